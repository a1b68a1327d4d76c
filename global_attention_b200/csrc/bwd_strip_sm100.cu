// bwd_strip_sm100.cu — query side of the gated sliding-window backward on tcgen05 / TMEM / TMA
// (sm_100a), organised by strips of positions like the forward (fwd_strip_sm100.cu).
//
// Exact gradients of L = sum(dout * out) for the ZGCM-1 layer (definition and page citations
// in common.cuh); this kernel forms, for W <= 128 and 4 query heads per KV head:
//   Delta_i = sum_j P_ij dP_ij,   dS = P (dP - Delta),   dq = RMSNorm/RoPE backward of scale dS K~
// and leaves Delta and the forward's lse (base 2) in the padded per-row arrays the key-major
// kernel (bwd_kv_tc_kernel) loads.  dA (fp16, row-scaled) comes from the gate pass, Q~ and K~
// (fp16) from the forward's activation store or the preparation kernels, V (fp16, one scale per
// 128-row tile) from the V preparation.
//
// A strip is (batch b, KV head, 32 positions p0..p0+31) with the group's 4 query heads: 128 MMA
// rows, row = 4 pos + head, whose windows all lie in the keys p0-128 .. p0+31 (five 32-key
// chunks).  Per strip:
//   S  = Q~ K~_span^T,  dP = dA V_span^T     tcgen05.mma M=128 N=160 K=128 each (fp16)
//   pass 1 (thread = row): P = 2^(S c - lse2) from the forward's lse, P dP written back over
//          S and dP, Delta = sum P dP, max |P dP|, and the RMSNorm row sums sum P dP S, sum P S
//   pass 2: dS = (P dP - P Delta) 2^e (fp16, e from max|P dP| + |Delta|) over the front of S
//   dQ~ = dS K~_span                          tcgen05.mma M=128 N=128 K=160, dS from TMEM
//   epilogue: RoPE / RMSNorm backward of the row (one pass over the raw q row), d_gamma_q
// TMEM: S [0,160), dP [160,320), dQ [320,448).  The next strip's S and dP are issued right
// after this strip's dQ, so the tensor core runs them while the epilogue drains dQ.
//
// Warp roles (512 threads): w0 TMA producer, w1 MMA issuer + TMEM owner, w2-3 idle, w4-7
// softmax passes, w8-11 idle, w12-15 dq epilogue.  Registers by warpgroup via setmaxnreg:
// 72 / 176 / 24 / 240 (the epilogue holds a whole dq~ row so it can release TMEM first).
// Every wait is bounded and voted warp-uniform where a warp-collective instruction follows;
// on expiry the CTA records the site, drains, frees TMEM and returns.
#include "bwd_tc.cuh"

namespace zgcm {

namespace {

constexpr int BSP = 32;                      // positions per strip
constexpr int BSG = 4;                       // query heads per KV head
constexpr int BNCH = 5;                      // 32-key chunks in a strip's window span
constexpr int BSPAN = BNCH * 32;             // 160
constexpr int BRING = 8;                     // chunk slots of the K~ / V rings
constexpr uint32_t BCH_HALF = 32 * 128;      // 32 rows x 64 dims (fp16): 4 KB
constexpr uint32_t BQ_HALF = 128 * 128;      // 128 rows x 64 dims: 16 KB
constexpr uint32_t BTM_S = 0, BTM_P = BSPAN, BTM_DQ = 2 * BSPAN;

enum SBar {
    SB_KF = 0, SB_VF = SB_KF + BRING, SB_KE = SB_VF + BRING,
    SB_QF = SB_KE + BRING, SB_QE, SB_SF, SB_DSF, SB_DQF, SB_DQE, SB_DONE, SB_COUNT
};

struct BwdStripSmem {
    alignas(1024) unsigned char K[2][BRING][BCH_HALF];    // [d-half][slot]: K~ fp16
    alignas(1024) unsigned char V[2][BRING][BCH_HALF];    // [d-half][slot]: V fp16 (tile-scaled)
    alignas(1024) unsigned char Q[2][BQ_HALF];            // Q~ fp16 of the strip
    alignas(1024) unsigned char dA[2][BQ_HALF];           // dA fp16 of the strip (row-scaled)
    float2 cs[BSP][TF_HALF];      // epilogue: (cos, sin) of the strip's positions
    float gq[kD], gk[kD];
    float dsinv[2][128];          // 2^-e of each dS row, by strip parity
    float mdot[2][128];           // mean(dy gamma xhat) of each row (RMSNorm backward), by parity
    float dgq[4][kD];             // this CTA's d_gamma_q, one slice per epilogue warp
    uint64_t bar[SB_COUNT];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(BwdStripSmem) + 1024 <= 227 * 1024, "strip backward shared memory over 227 KB");

struct BStrip {
    int b, kvh, s;
    bool fresh;
};

__device__ __forceinline__ BStrip bstrip_at(const LayerParams& L, int nst, int t, int t_begin) {
    BStrip st;
    const int chain = t / nst;
    st.s = t - chain * nst;
    st.b = chain / L.Hkv;
    st.kvh = chain - st.b * L.Hkv;
    st.fresh = (t == t_begin) || (st.s == 0);
    return st;
}

// S = Q~ K~^T and dP = dA V^T over the span's ring slots (one run, or two around the ring's
// end), K-step by K-step: the two (or four) independent accumulation chains are issued in
// turn, so the tensor pipe overlaps them instead of waiting on each dependent step.
__device__ __forceinline__ void issue_s_dp(uint32_t tS, uint32_t tP, uint64_t q_desc, uint64_t da_desc,
                                           uint64_t k_desc0, uint64_t v_desc0, int s0, int run0, int nch) {
    const uint32_t id0 = idesc_f16(128, 32 * run0, false), id1 = idesc_f16(128, 32 * (nch - run0), false);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t half = kk >> 2, within = (kk & 3) * 32;
        const uint32_t ao = half * BQ_HALF + within, bo = half * BRING * BCH_HALF + within;
        const uint32_t acc = kk > 0 ? 1u : 0u;
        mma_ss(tS, sdesc_step(q_desc, ao), sdesc_step(k_desc0, s0 * BCH_HALF + bo), id0, acc);
        mma_ss(tP, sdesc_step(da_desc, ao), sdesc_step(v_desc0, s0 * BCH_HALF + bo), id0, acc);
        if (run0 < nch) {
            mma_ss(tS + 32 * run0, sdesc_step(q_desc, ao), sdesc_step(k_desc0, bo), id1, acc);
            mma_ss(tP + 32 * run0, sdesc_step(da_desc, ao), sdesc_step(v_desc0, bo), id1, acc);
        }
    }
}

// Pass 1 over one 32-key chunk of a row (vm: visible keys; ignored when FULL)
template <bool FULL>
__device__ __forceinline__ void strip_pass1(float (&sv)[32], float (&dv)[32], uint32_t vm, float c2, float lse2,
                                            float& cnum, float& cmpd, float& csa, float& sb) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const float s = sv[e];
        float pv = fast_exp2(fmaf(s, c2, -lse2));
        if (!FULL) pv = ((vm >> e) & 1u) ? pv : 0.f;  // (a masked score may overflow: selected away)
        const float pd = pv * dv[e];
        cnum += pd;
        cmpd = fmaxf(cmpd, fabsf(pd));
        csa = fmaf(pd, s, csa);
        sb = fmaf(pv, s, sb);
        sv[e] = pv;
        dv[e] = pd;
    }
}

}  // namespace

__global__ void __launch_bounds__(TB_THREADS, 1) bwd_strip_q_kernel(const __grid_constant__ BwdTcParams p) {
    const LayerParams& L = p.P.L;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    BwdStripSmem& sm =
        *reinterpret_cast<BwdStripSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &sm.abort;
    const int nst = (L.S + BSP - 1) / BSP;
    const int t_begin = (int)(((long long)blockIdx.x * p.total) / gridDim.x);
    const int t_end = (int)(((long long)(blockIdx.x + 1) * p.total) / gridDim.x);
    const int nstrips = t_end - t_begin;

    if (tid == 0) {
        sm.abort = 0;
        for (int i = 0; i < BRING; ++i) {
            mbar_init(&sm.bar[SB_KF + i], 1);
            mbar_init(&sm.bar[SB_VF + i], 1);
            mbar_init(&sm.bar[SB_KE + i], 1);
        }
        mbar_init(&sm.bar[SB_QF], 1);
        mbar_init(&sm.bar[SB_QE], 1);
        mbar_init(&sm.bar[SB_SF], 1);
        mbar_init(&sm.bar[SB_DSF], 128);
        mbar_init(&sm.bar[SB_DQF], 1);
        mbar_init(&sm.bar[SB_DQE], 128);
        mbar_init(&sm.bar[SB_DONE], 1);
        fence_barrier_init();
    }
    if (tid < kD) {
        sm.gq[tid] = L.gamma_q[tid];
        sm.gk[tid] = L.gamma_k[tid];
        for (int w = 0; w < 4; ++w) sm.dgq[w][tid] = 0.f;
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tm_q16s);
        prefetch_tmap(&p.tm_das);
        prefetch_tmap(&p.tm_k16c);
        prefetch_tmap(&p.tm_v16c);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    const float c2 = L.scale_log2 / (oscale * oscale);
    const float mdot_f = c2 * kLn2 / (float)kD;  // scale / (D oscale^2)

    if (warp < 4) {
        reg_dealloc<72>();
        if (warp == 0 && lane == 0) {
            // ================================================ TMA producer
            // Q~ and dA of a strip (one buffer each), K~ and V chunks (8-slot ring); the two
            // streams are polled so that neither blocks the other.
            int nq = 0, tq = t_begin, lk = 0, tk = t_begin, ck = 0, nck = 0;
            BStrip stk{};
            int last_q = -1, last_l[BRING];
            for (int i = 0; i < BRING; ++i) last_l[i] = -1;
            uint32_t idle = 0;
            while ((nq < nstrips || tk < t_end) && !*abort) {
                bool moved = false;
                if (nq < nstrips && (nq == 0 || mbar_try_wait(&sm.bar[SB_QE], (nq - 1) & 1))) {
                    const BStrip st = bstrip_at(L, nst, tq, t_begin);
                    mbar_expect_tx(&sm.bar[SB_QF], 4 * BQ_HALF);
                    tma_load_4d(sm.Q[0], &p.tm_q16s, &sm.bar[SB_QF], 0, st.kvh * BSG, st.s * BSP, st.b);
                    tma_load_4d(sm.Q[1], &p.tm_q16s, &sm.bar[SB_QF], 64, st.kvh * BSG, st.s * BSP, st.b);
                    tma_load_4d(sm.dA[0], &p.tm_das, &sm.bar[SB_QF], 0, st.kvh * BSG, st.s * BSP, st.b);
                    tma_load_4d(sm.dA[1], &p.tm_das, &sm.bar[SB_QF], 64, st.kvh * BSG, st.s * BSP, st.b);
                    last_q = nq;
                    ++nq;
                    ++tq;
                    moved = true;
                }
                if (tk < t_end) {
                    if (nck == 0) {
                        stk = bstrip_at(L, nst, tk, t_begin);
                        nck = stk.fresh ? BNCH : 1;
                        ck = stk.s - nck + 1;
                    }
                    const int slot = lk % BRING;
                    if (lk < BRING || mbar_try_wait(&sm.bar[SB_KE + slot], ((lk / BRING) - 1) & 1)) {
                        mbar_expect_tx(&sm.bar[SB_KF + slot], 2 * BCH_HALF);
                        tma_load_4d(sm.K[0][slot], &p.tm_k16c, &sm.bar[SB_KF + slot], 0, stk.kvh, ck * 32, stk.b);
                        tma_load_4d(sm.K[1][slot], &p.tm_k16c, &sm.bar[SB_KF + slot], 64, stk.kvh, ck * 32, stk.b);
                        mbar_expect_tx(&sm.bar[SB_VF + slot], 2 * BCH_HALF);
                        tma_load_4d(sm.V[0][slot], &p.tm_v16c, &sm.bar[SB_VF + slot], 0, stk.kvh, ck * 32, stk.b);
                        tma_load_4d(sm.V[1][slot], &p.tm_v16c, &sm.bar[SB_VF + slot], 64, stk.kvh, ck * 32, stk.b);
                        last_l[slot] = lk;
                        ++lk;
                        ++ck;
                        if (--nck == 0) ++tk;
                        moved = true;
                    }
                }
                if (moved) {
                    idle = 0;
                } else if (++idle > kWaitLimit) {
                    *abort = 301;
                    break;
                }
            }
            if (last_q >= 0) mbar_wait_drain(&sm.bar[SB_QF], last_q & 1);
            for (int sl = 0; sl < BRING; ++sl)
                if (last_l[sl] >= 0) {
                    mbar_wait_drain(&sm.bar[SB_KF + sl], (last_l[sl] / BRING) & 1);
                    mbar_wait_drain(&sm.bar[SB_VF + sl], (last_l[sl] / BRING) & 1);
                }
        } else if (warp == 1 && lane == 0) {
            // ================================================ MMA issuer
            constexpr uint32_t IDESC_DQ = idesc_f16(128, 128, true);
            const uint64_t q_d = sdesc_sw128(smem_u32(sm.Q[0]), 16, 1024);
            const uint64_t da_d = sdesc_sw128(smem_u32(sm.dA[0]), 16, 1024);
            const uint64_t k_d = sdesc_sw128(smem_u32(sm.K[0][0]), 16, 1024);
            const uint64_t v_d = sdesc_sw128(smem_u32(sm.V[0][0]), 16, 1024);
            const uint64_t k_mn = sdesc_sw128(smem_u32(sm.K[0][0]), BRING * BCH_HALF, 1024);
            int lcount = 0, kwait = 0;
            bool ok = true;
            int le_prev = -1;
            auto issue_dq = [&](int m, int le, int le_next) -> bool {
                // dS of strip m is in TMEM once the softmax arrives; dQ waits for the epilogue
                // to have read the previous strip's dQ
                if (!mbar_wait(&sm.bar[SB_DSF], m & 1, abort, 310)) return false;
                if (m >= 1 && !mbar_wait(&sm.bar[SB_DQE], (m - 1) & 1, abort, 311)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 2 * BNCH; ++kk) {
                    const int slot = (le - (BNCH - 1) + (kk >> 1)) % BRING;
                    mma_ts(tmem + BTM_DQ, tmem + BTM_S + kk * 8, sdesc_step(k_mn, slot * BCH_HALF + (kk & 1) * 2048),
                           IDESC_DQ, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar[SB_DQF]);
                // chunks no later strip reads
                const int keep_from = le_next < 0 ? le + 1 : le_next - (BNCH - 1);
                for (int l = le - (BNCH - 1); l <= le && l < keep_from; ++l) mma_commit(&sm.bar[SB_KE + l % BRING]);
                return true;
            };
            for (int n = 0; n < nstrips && ok; ++n) {
                const BStrip st = bstrip_at(L, nst, t_begin + n, t_begin);
                lcount += st.fresh ? BNCH : 1;
                const int le = lcount - 1;
                if (n >= 1 && !(ok = issue_dq(n - 1, le_prev, le))) break;
                if (!(ok = mbar_wait(&sm.bar[SB_QF], n & 1, abort, 312))) break;
                for (; kwait <= le && ok; ++kwait)
                    ok = mbar_wait(&sm.bar[SB_KF + kwait % BRING], (kwait / BRING) & 1, abort, 313) &&
                         mbar_wait(&sm.bar[SB_VF + kwait % BRING], (kwait / BRING) & 1, abort, 314);
                if (!ok) break;
                tc_fence_after();
                const int s0 = (le - (BNCH - 1)) % BRING;
                const int run0 = min(BNCH, BRING - s0);
                issue_s_dp(tmem + BTM_S, tmem + BTM_P, q_d, da_d, k_d, v_d, s0, run0, BNCH);
                mma_commit(&sm.bar[SB_QE]);
                mma_commit(&sm.bar[SB_SF]);
                le_prev = le;
            }
            if (ok && nstrips > 0) issue_dq(nstrips - 1, le_prev, -1);
            mma_commit(&sm.bar[SB_DONE]);
            mbar_wait_drain(&sm.bar[SB_DONE], 0);
        }
    } else if (warp < 8) {
        reg_alloc<176>();
        // ================================================ Delta, dS (thread = row 4 pos + head)
        const int m = tid - 128, pos = m >> 2;
        const int Spad = row_stride(L.S), nkt = (L.S + TF_BN - 1) / TF_BN;
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        for (int n = 0; n < nstrips; ++n) {
            const BStrip st = bstrip_at(L, nst, t_begin + n, t_begin);
            const int p0 = st.s * BSP, i = p0 + pos, h = st.kvh * BSG + (m & 3);
            const bool valid = i < L.S;
            const size_t ro = ((size_t)st.b * L.Hq + h) * L.S + (valid ? i : 0);
            const size_t rbase = ((size_t)st.b * L.Hq + h) * Spad;
            const float lse2 = valid ? p.P.lse[ro] * kLog2e : INFINITY;
            const float dai = valid ? p.dainv[rbase + i] : 0.f;
            // visible span offsets o (key p0 - 128 + o): i - W < key <= i, key >= 0
            const int olo = max(max(pos + 129 - L.W, 128 - p0), 0), ohi = pos + 128;
            // dP = (accumulated) * dainv * V tile scale: one factor per chunk (chunks before
            // the sequence start hold no key)
            const float* vtrow = p.vtinv + ((size_t)st.b * L.Hkv + st.kvh) * nkt;
            float kd[BNCH];
#pragma unroll
            for (int c = 0; c < BNCH; ++c) {
                const int key0 = p0 - 128 + 32 * c;
                kd[c] = key0 >= 0 ? dai * vtrow[key0 / TF_BN] : 0.f;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar[SB_SF], n & 1, abort, 320))) break;
            tc_fence_after();
            float num = 0.f, mpd = 0.f, sa = 0.f, sb = 0.f;
#pragma unroll 1
            for (int c = 0; c < BNCH; ++c) {
                const uint32_t vm = bit_range(olo - 32 * c, ohi - 32 * c);
                if (__all_sync(0xffffffffu, vm == 0u)) continue;
                float sv[32], dv[32];
                tmem_ld32f(tmem + BTM_S + lane_off + 32 * c, sv);
                tmem_ld32f(tmem + BTM_P + lane_off + 32 * c, dv);
                tmem_wait_ld();
                float cnum = 0.f, cmpd = 0.f, csa = 0.f;
                if (__all_sync(0xffffffffu, vm == 0xffffffffu))
                    strip_pass1<true>(sv, dv, 0u, c2, lse2, cnum, cmpd, csa, sb);
                else
                    strip_pass1<false>(sv, dv, vm, c2, lse2, cnum, cmpd, csa, sb);
                num = fmaf(kd[c], cnum, num);
                mpd = fmaxf(mpd, fabsf(kd[c]) * cmpd);
                sa = fmaf(kd[c], csa, sa);
                tmem_st32f(tmem + BTM_S + lane_off + 32 * c, sv);
                tmem_st32f(tmem + BTM_P + lane_off + 32 * c, dv);
            }
            tmem_wait_st();
            const float delta = num;
            // |dS| = |P dP - P Delta| <= max |P dP| + |Delta|
            const float dsc = ldexpf(1.0f, fit_exp(mpd + fabsf(delta)));
#pragma unroll 1
            for (int c = 0; c < BNCH; ++c) {
                const uint32_t vm = bit_range(olo - 32 * c, ohi - 32 * c);
                uint32_t pk[16];
                if (!__all_sync(0xffffffffu, vm == 0u)) {
                    float pv[32], pd[32];
                    tmem_ld32f(tmem + BTM_S + lane_off + 32 * c, pv);
                    tmem_ld32f(tmem + BTM_P + lane_off + 32 * c, pd);
                    tmem_wait_ld();
                    // pd holds P dv: dS dsc = P dv (kd dsc) - P (Delta dsc)
                    const float ka = kd[c] * dsc, kb = -delta * dsc;
                    const float2 ka2 = make_float2(ka, ka), kb2 = make_float2(kb, kb);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float2 t = ffma2(make_float2(pd[e], pd[e + 1]), ka2,
                                               fmul2(make_float2(pv[e], pv[e + 1]), kb2));
                        pk[e >> 1] = pack2<true>(t.x, t.y);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                }
                tmem_st16(tmem + BTM_S + lane_off + 16 * c, pk);
            }
            tmem_wait_st();
            sm.dsinv[n & 1][m] = 1.0f / dsc;
            sm.mdot[n & 1][m] = fmaf(-delta, sb, sa) * mdot_f;  // sum dS S = a - Delta b
            tc_fence_before();
            mbar_arrive(&sm.bar[SB_DSF]);
            // Delta and the base-2 lse per row for the key-major kernel; the rows past S up to
            // the padded length get the neutral values (P = 0 there, dA scale 0)
            if (valid) {
                p.P.delta[rbase + i] = delta;
                p.lse2p[rbase + i] = lse2;
            } else if (i < Spad) {
                p.P.delta[rbase + i] = 0.f;
                p.lse2p[rbase + i] = INFINITY;
                p.dainv[rbase + i] = 0.f;
            }
            if (st.s == nst - 1 && i + BSP >= L.S && i + BSP < Spad) {
                p.P.delta[rbase + i + BSP] = 0.f;
                p.lse2p[rbase + i + BSP] = INFINITY;
                p.dainv[rbase + i + BSP] = 0.f;
            }
        }
    } else if (warp < 12) {
        reg_dealloc<24>();
    } else {
        reg_alloc<240>();
        // ================================================ dq epilogue (thread = row 4 pos + head)
        const int m = tid - 384, pos = m >> 2, wq = warp - 12;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        for (int n = 0; n < nstrips; ++n) {
            const BStrip st = bstrip_at(L, nst, t_begin + n, t_begin);
            const int p0 = st.s * BSP, i = p0 + pos, h = st.kvh * BSG + (m & 3);
            const bool valid = i < L.S;
            // rotation angles of the warp's 8 positions (4 threads per position)
            __syncwarp();
            for (int q = m & 3; q < TF_HALF; q += 4) {
                float2 w;
                rope_cs(L.theta[q], i, w.x, w.y);
                sm.cs[pos][q] = w;
            }
            __syncwarp();
            const size_t off = ((size_t)(st.b * (size_t)L.S + (valid ? i : 0)) * L.Hq + h) * kD;
            const float rinv = valid ? p.qrinv[((size_t)st.b * L.Hq + h) * L.S + i] : 0.f;
            uint4 xv0[8];  // first half of the raw q row, in flight during the wait
#pragma unroll
            for (int c = 0; c < 8; ++c)
                xv0[c] = valid ? __ldg(reinterpret_cast<const uint4*>(L.q + off) + c) : make_uint4(0u, 0u, 0u, 0u);
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar[SB_DQF], n & 1, abort, 330))) break;
            tc_fence_after();
            float dy[128];
            const uint32_t tq = tmem + BTM_DQ + lane_off;
            tmem_ld32f(tq, dy);
            tmem_ld32f(tq + 32, dy + 32);
            tmem_ld32f(tq + 64, dy + 64);
            tmem_ld32f(tq + 96, dy + 96);
            tmem_wait_ld();
            const float f = L.scale * sm.dsinv[n & 1][m] / oscale;
            const float mdot = sm.mdot[n & 1][m];
            tc_fence_before();
            mbar_arrive(&sm.bar[SB_DQE]);  // dQ is in registers: TMEM free for the next dQ
            row_rope_rms_backward_cs(dy, f, mdot, rinv, xv0, L.q + off, p.P.dq + off, valid,
                                     [&](int q) { return sm.cs[pos][q]; }, sm.gq, sm.dgq[wq]);
        }
    }

    // ------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
    if (tid < kD)
        p.P.dgq_part[(size_t)blockIdx.x * kD + tid] = (sm.dgq[0][tid] + sm.dgq[1][tid]) + (sm.dgq[2][tid] + sm.dgq[3][tid]);
    if (tid == 0 && sm.abort && p.err) atomicExch(p.err, sm.abort);
}

// 4 query heads per KV head (the strip's 128 rows), windows up to 128, 42 rotated dims.
bool bwd_strip_supported(const LayerParams& L) {
    return L.W <= TF_BN && L.G == BSG && L.rope_half == TF_HALF && L.S >= 1 && L.B >= 1;
}

size_t bwd_strip_smem_bytes() { return sizeof(BwdStripSmem) + 1024; }

int bwd_strip_total(const LayerParams& L) {
    const long long t = (long long)L.B * L.Hkv * ((L.S + BSP - 1) / BSP);
    return t > 0x7fffffffLL ? -1 : (int)t;
}

}  // namespace zgcm
