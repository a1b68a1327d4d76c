// bwd_glob_sm100.cu — backward pieces for windows wider than one key tile: the full-causal
// global layer (W >= S; ZGCM-1 layers 6/12/18/24/30) and any W > 128, on tcgen05 / TMEM /
// TMA (sm_100a).  Layer definition and page citations: common.cuh.
//
// The wide-window backward runs the gate pass (which also writes Delta_i = sum_d dout*out,
// the row sum of dA * A, since A = out / sigmoid(g) and dA = dout * sigmoid(g)), the Q / K / V
// preparation, then:
//   bwd_tile_stats_kernel  per (b, KV head, 128-row tile): max |dout| and max |Delta| over the
//                          tile's rows of the group's query heads, and max ||v|| over its key
//                          rows.  The fp16 scales below come from these bounds, known before
//                          any product, because a row's dS feeds an accumulator that spans
//                          all of its key tiles.
//   bwd_q_glob_kernel      query-major: one CTA per (b, query head, 128-query block), heaviest
//                          blocks first, sweeping the key tiles of the window:
//                            S  = Q~ K~^T, dP = dA V^T     (M=128, N=128, K=128; TMEM)
//                            dS = P (dP - Delta), P = 2^(S c2 - lse2) with the forward's lse
//                            dQ~ += dS K~                  (dS fp16 from TMEM, K~ MN-major)
//                          then the RoPE / RMSNorm backward writes dq.
//   bwd_kv_tc_kernel       the sliding-window key-major kernel in its one-unit-per-CTA mode
//                          (dK, dV, GQA sums; bwd_sm100.cu).
#include "bwd_tc.cuh"

namespace zgcm {

// =====================================================================  tile statistics

// One CTA of 128 threads per (b, KV head, tile t): thread r takes query row t*128 + r of each
// head of the group and key row t*128 + r.  Writes p.tstat[k][(b*Hkv + kvh)*ntile + t] for
// k = 0 (max |dout|), 1 (max |Delta|), 2 (max ||v||); rows past S, and query rows before the
// first one (q_off), contribute 0.
__global__ void __launch_bounds__(BTS_THREADS) bwd_tile_stats_kernel(const __grid_constant__ BwdTcParams p) {
    const LayerParams& L = p.P.L;
    const int r = threadIdx.x, lane = r & 31, warp = r >> 5;
    const int nt = (L.S + TF_BN - 1) / TF_BN, Spad = row_stride(L.S);
    const int t = (int)blockIdx.x % nt, chain = (int)blockIdx.x / nt;
    const int kvh = chain % L.Hkv, b = chain / L.Hkv;
    const int i = t * TF_BN + r;
    float dm = 0.f, dl = 0.f, vn = 0.f;
    if (i < L.S) {
        for (int h = 0; h < L.G && i >= L.q_off; ++h) {
            const size_t rp = ((size_t)b * L.Hq + kvh * L.G + h) * Spad + i;
            dm = fmaxf(dm, p.domax[rp]);
            dl = fmaxf(dl, fabsf(p.P.delta[rp]));
        }
        vn = p.vnorm[((size_t)b * L.Hkv + kvh) * L.S + i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        dm = fmaxf(dm, __shfl_xor_sync(0xffffffffu, dm, o));
        dl = fmaxf(dl, __shfl_xor_sync(0xffffffffu, dl, o));
        vn = fmaxf(vn, __shfl_xor_sync(0xffffffffu, vn, o));
    }
    __shared__ float red[3][4];
    if (lane == 0) {
        red[0][warp] = dm;
        red[1][warp] = dl;
        red[2][warp] = vn;
    }
    __syncthreads();
    if (r < 3) {
        const size_t n = (size_t)L.B * L.Hkv * nt;
        p.tstat[(size_t)r * n + (size_t)chain * nt + t] =
            fmaxf(fmaxf(red[r][0], red[r][1]), fmaxf(red[r][2], red[r][3]));
    }
}

// =====================================================================  query-major kernel

constexpr int QG_KSLOTS = 3;   // K~ ring (read by S(n) and, one iteration later, by dQ(n))
constexpr int QG_VSLOTS = 2;   // V ring (read by dP(n) only)

enum QgBar {
    QG_QFULL = 0,                              // Q~ and dA of the unit
    QG_KFULL = 1, QG_KEMPTY = QG_KFULL + QG_KSLOTS,
    QG_VFULL = QG_KEMPTY + QG_KSLOTS, QG_VEMPTY = QG_VFULL + QG_VSLOTS,
    QG_SDPFULL = QG_VEMPTY + QG_VSLOTS,        // S(n) and dP(n) in TMEM
    QG_DPFREE = QG_SDPFULL + 1,                // both softmax warpgroups have read dP(n)
    QG_DSFULL = QG_DPFREE + 1,                 // dS(n) (fp16) in TMEM
    QG_DQFULL = QG_DSFULL + 1,                 // every product done: dQ~ final
    QG_MDOT = QG_DQFULL + 1,                   // the second warpgroup's RMSNorm row sums
    QG_DELTA = QG_MDOT + 1,                    // both halves of a one-tile sweep's sum P dP
    QG_DQDONE = QG_DELTA + 1,                  // dQ(n) has read dS(n): S buffer n % 2 free (2)
    QG_SDONE = QG_DQDONE + 2,                  // the S / dP issuer's products are complete
    QG_COUNT = QG_SDONE + 1
};

struct BwdQGlobSmem {
    alignas(1024) unsigned char Q[2][TF_HALF_BYTES];               // Q~ fp16 of the unit
    alignas(1024) unsigned char dA[2][TF_HALF_BYTES];              // dA fp16, row-scaled
    alignas(1024) unsigned char K[QG_KSLOTS][2][TF_HALF_BYTES];    // K~ fp16 ring
    // V fp16 ring (tile-scaled).  Slot 1 also holds, where it is idle: a one-tile sweep's
    // sums of P dP over each 64-key half (dpart [2][128], during the tile: the sweep loads no
    // V there) and, after the sweep, the second warpgroup's sums dS S (mdot_hi [128], at 1 KB);
    // slot 0 the d_gamma slices of the epilogue warps.
    alignas(1024) unsigned char V[QG_VSLOTS][2][TF_HALF_BYTES];
    float gq[kD], gk[kD];
    uint64_t bar[QG_COUNT];
    uint32_t tmem_base;
    int abort;
};

// (+1024: the kernel aligns the dynamic shared memory to 1 KB itself)
static_assert(sizeof(BwdQGlobSmem) + 1024 <= 232448, "beyond the 227 KB of shared memory a CTA can have");
size_t bwd_q_glob_smem_bytes() { return sizeof(BwdQGlobSmem) + 1024; }

// dS of 32 keys of a row, already times its power-of-two scale dsc (kds = kd dsc, dls =
// Delta dsc: a power-of-two factor commutes with every rounding, so these are the values
// (P (dP kd - Delta)) dsc exactly), packed to fp16; ma[] accumulates (dS dsc) S in two
// partials.  MASK: keys outside the row's window (vm) get P = 0.
template <bool MASK>
__device__ __forceinline__ void qg_ds_chunk(const float* sv, const float* dv, uint32_t vm, float c2, float lse2,
                                            float kds, float dls, float (&ma)[2], uint32_t (&pk)[16]) {
    // two keys per paired fp32 instruction
    const float2 cc = make_float2(c2, c2), nl = make_float2(-lse2, -lse2);
    const float2 kk = make_float2(kds, kds), nd = make_float2(-dls, -dls);
    float2 acc = make_float2(ma[0], ma[1]);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const float2 s = make_float2(sv[e], sv[e + 1]);
        const float2 x = ffma2(s, cc, nl);
        float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
        if (MASK) {
            p.x = ((vm >> e) & 1u) ? p.x : 0.f;  // (a masked score may overflow: selected away)
            p.y = ((vm >> (e + 1)) & 1u) ? p.y : 0.f;
        }
        const float2 d = fmul2(p, ffma2(make_float2(dv[e], dv[e + 1]), kk, nd));
        acc = ffma2(d, s, acc);
        pk[e >> 1] = pack2<true>(d.x, d.y);
    }
    ma[0] = acc.x;
    ma[1] = acc.y;
}

// ANY: any number of rotated pairs in the dq epilogue (else the layer's 21, unrolled)
template <bool ANY>
__global__ void __launch_bounds__(BQG_THREADS, 1) bwd_q_glob_kernel(const __grid_constant__ BwdTcParams p) {
    const LayerParams& L = p.P.L;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    BwdQGlobSmem& sm = *reinterpret_cast<BwdQGlobSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &sm.abort;
    // unit, heaviest first: block qb from the last one down (to the block of the first query
    // row, q_off / 128: the launcher's unit count), then batch and head
    const int nqb = (L.S + TF_BM - 1) / TF_BM, nkt = nqb;
    const int per_qb = L.B * L.Hq;
    const int u = (int)blockIdx.x;
    const int qb = nqb - 1 - u / per_qb, rest = u % per_qb;
    const int b = rest / L.Hq, hq = rest % L.Hq, kvh = hq / L.G;
    const int q0 = qb * TF_BM;
    const int kt_lo = (L.W >= L.S || q0 - L.W + 1 <= 0) ? 0 : (q0 - L.W + 1) / TF_BN;
    const int N = qb - kt_lo + 1;  // key tiles of the sweep

    if (tid == 0) {
        sm.abort = 0;
        mbar_init(&sm.bar[QG_QFULL], 1);
        for (int s = 0; s < QG_KSLOTS; ++s) {
            mbar_init(&sm.bar[QG_KFULL + s], 1);
            mbar_init(&sm.bar[QG_KEMPTY + s], 1);
        }
        for (int s = 0; s < QG_VSLOTS; ++s) {
            mbar_init(&sm.bar[QG_VFULL + s], 1);
            mbar_init(&sm.bar[QG_VEMPTY + s], 1);
        }
        mbar_init(&sm.bar[QG_SDPFULL], 1);
        mbar_init(&sm.bar[QG_DPFREE], 256);
        mbar_init(&sm.bar[QG_DSFULL], 256);
        mbar_init(&sm.bar[QG_DQFULL], 1);
        mbar_init(&sm.bar[QG_MDOT], 128);
        mbar_init(&sm.bar[QG_DELTA], 256);
        mbar_init(&sm.bar[QG_DQDONE], 1);
        mbar_init(&sm.bar[QG_DQDONE + 1], 1);
        mbar_init(&sm.bar[QG_SDONE], 1);
        fence_barrier_init();
    }
    if (tid < kD) {
        sm.gq[tid] = L.gamma_q[tid];
        sm.gk[tid] = L.gamma_k[tid];
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tm_q16);
        prefetch_tmap(&p.tm_da);
        prefetch_tmap(&p.tm_k16);
        prefetch_tmap(&p.tm_v16);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // TMEM: S(n) in [128 (n%2), +128); dP(n) in [256, 384); dQ~ in [384, 512).  dS(n) (fp16)
    // goes over S(n): keys 0-63 at columns [0, 32), keys 64-127 at [64, 96), each half inside
    // the columns its own warpgroup read, so neither overwrites scores the other still reads.
    const uint32_t TM_DP = tmem + 256, TM_DQ = tmem + 384;
    auto tm_s = [&](int n) -> uint32_t { return tmem + 128u * (uint32_t)(n & 1); };
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    const float c2 = L.scale_log2 / (oscale * oscale);
    const float mdot_f = c2 * kLn2 / (float)kD;  // scale / (D oscale^2)

    // registers (set inside each role's branch): warpgroup 0 56, softmax + epilogue 232,
    // softmax 216; 128 * (56 + 232 + 216) = 384 * 168, the launch's allocation
    if (warp == 0) {
        // ================================================ TMA producer
        reg_dealloc<56>();
        if (lane == 0) {
            mbar_expect_tx(&sm.bar[QG_QFULL], 2 * TF_TILE_BYTES);
            tma_load_4d(sm.Q[0], &p.tm_q16, &sm.bar[QG_QFULL], 0, hq, q0, b);
            tma_load_4d(sm.Q[1], &p.tm_q16, &sm.bar[QG_QFULL], 64, hq, q0, b);
            tma_load_4d(sm.dA[0], &p.tm_da, &sm.bar[QG_QFULL], 0, hq, q0, b);
            tma_load_4d(sm.dA[1], &p.tm_da, &sm.bar[QG_QFULL], 64, hq, q0, b);
            int nk = 0, nv = 0;
            for (int n = 0; n < N; ++n) {
                const int k0 = (kt_lo + n) * TF_BN;
                const int ks = n % QG_KSLOTS, vs = n % QG_VSLOTS;
                if (n >= QG_KSLOTS && !mbar_wait(&sm.bar[QG_KEMPTY + ks], ((n / QG_KSLOTS) & 1) ^ 1, abort, 300)) break;
                mbar_expect_tx(&sm.bar[QG_KFULL + ks], TF_TILE_BYTES);
                tma_load_4d(sm.K[ks][0], &p.tm_k16, &sm.bar[QG_KFULL + ks], 0, kvh, k0, b);
                tma_load_4d(sm.K[ks][1], &p.tm_k16, &sm.bar[QG_KFULL + ks], 64, kvh, k0, b);
                nk = n + 1;
                if (n >= QG_VSLOTS && !mbar_wait(&sm.bar[QG_VEMPTY + vs], ((n / QG_VSLOTS) & 1) ^ 1, abort, 301)) break;
                mbar_expect_tx(&sm.bar[QG_VFULL + vs], TF_TILE_BYTES);
                tma_load_4d(sm.V[vs][0], &p.tm_v16, &sm.bar[QG_VFULL + vs], 0, kvh, k0, b);
                tma_load_4d(sm.V[vs][1], &p.tm_v16, &sm.bar[QG_VFULL + vs], 64, kvh, k0, b);
                nv = n + 1;
            }
            // every copy issued must land before the CTA exits (matters after an abort)
            mbar_wait_drain(&sm.bar[QG_QFULL], 0);
            for (int n = nk > QG_KSLOTS ? nk - QG_KSLOTS : 0; n < nk; ++n)
                mbar_wait_drain(&sm.bar[QG_KFULL + n % QG_KSLOTS], (n / QG_KSLOTS) & 1);
            for (int n = nv > QG_VSLOTS ? nv - QG_VSLOTS : 0; n < nv; ++n)
                mbar_wait_drain(&sm.bar[QG_VFULL + n % QG_VSLOTS], (n / QG_VSLOTS) & 1);
        }
    } else if (warp == 1 || warp == 2) {
        // ================================================ MMA issuers
        // warp 1: S(0) dP(0) S(1), then per tile n: dP(n+1) once dP(n) has been read, S(n+2)
        // over S(n) once dQ(n), which reads dS(n) there, has completed (QG_DQDONE);
        // warp 2: dQ(n) once dS(n) is written.  Two issuing threads, so that neither one's
        // waits leave the tensor pipe without instructions.
        reg_dealloc<56>();
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_f16(128, 128, false);
            constexpr uint32_t IDESC_DQ = idesc_f16(128, 128, true);
            const uint32_t q_base = smem_u32(sm.Q[0]), da_base = smem_u32(sm.dA[0]);
            const uint32_t k_base = smem_u32(sm.K[0][0]), v_base = smem_u32(sm.V[0][0]);
            auto issue_s = [&](int n) {
                const uint32_t kb = k_base + (uint32_t)(n % QG_KSLOTS) * 2u * TF_HALF_BYTES;
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * TF_HALF_BYTES + (kk & 3) * 32;
                    mma_ss(tm_s(n), sdesc_sw128(q_base + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), IDESC_S,
                           kk > 0 ? 1u : 0u);
                }
            };
            auto issue_dp = [&](int n) {
                const uint32_t vb = v_base + (uint32_t)(n % QG_VSLOTS) * 2u * TF_HALF_BYTES;
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * TF_HALF_BYTES + (kk & 3) * 32;
                    mma_ss(TM_DP, sdesc_sw128(da_base + off, 16, 1024), sdesc_sw128(vb + off, 16, 1024), IDESC_S,
                           kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar[QG_SDPFULL]);
                mma_commit(&sm.bar[QG_VEMPTY + n % QG_VSLOTS]);
            };
            auto issue_dq = [&](int n) {
                const uint32_t kb = k_base + (uint32_t)(n % QG_KSLOTS) * 2u * TF_HALF_BYTES;
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    // 16 keys per step: dS columns 8 kk (keys 0-63) or 64 + 8 (kk - 4) (keys 64-127)
                    const uint32_t acol = kk < 4 ? 8u * kk : 64u + 8u * (kk - 4);
                    mma_ts(TM_DQ, tm_s(n) + acol, sdesc_sw128(kb + kk * 16 * 128, TF_HALF_BYTES, 1024), IDESC_DQ,
                           (n > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&sm.bar[QG_KEMPTY + n % QG_KSLOTS]);  // (S(n) completed before dS(n) existed)
                mma_commit(&sm.bar[QG_DQDONE + (n & 1)]);
            };
            auto kfull = [&](int n, int site) {
                return mbar_wait(&sm.bar[QG_KFULL + n % QG_KSLOTS], (n / QG_KSLOTS) & 1, abort, site);
            };
            auto vfull = [&](int n, int site) {
                return mbar_wait(&sm.bar[QG_VFULL + n % QG_VSLOTS], (n / QG_VSLOTS) & 1, abort, site);
            };
            if (warp == 2) {
                bool ok = true;
                for (int n = 0; n < N && ok; ++n) {
                    if (!(ok = mbar_wait(&sm.bar[QG_DSFULL], n & 1, abort, 316))) break;
                    tc_fence_after();
                    issue_dq(n);
                }
                // every MMA issued must complete before TMEM is released; DQFULL is that point
                // for the dQ products (the S / dP ones complete before the last dS exists)
                mma_commit(&sm.bar[QG_DQFULL]);
                if (!mbar_wait(&sm.bar[QG_DQFULL], 0, abort, 318)) mbar_wait_drain(&sm.bar[QG_DQFULL], 0);
            } else {
                bool ok = mbar_wait(&sm.bar[QG_QFULL], 0, abort, 310) && kfull(0, 311);
                if (ok) {
                    tc_fence_after();
                    issue_s(0);
                    ok = vfull(0, 312);
                }
                if (ok) {
                    tc_fence_after();
                    issue_dp(0);
                    if (N > 1 && (ok = kfull(1, 313))) {
                        tc_fence_after();
                        issue_s(1);
                    }
                }
                for (int n = 0; n < N && ok; ++n) {
                    if (n + 1 < N) {
                        if (!(ok = mbar_wait(&sm.bar[QG_DPFREE], n & 1, abort, 314) && vfull(n + 1, 315))) break;
                        tc_fence_after();
                        issue_dp(n + 1);
                    }
                    if (n + 2 < N) {
                        if (!(ok = mbar_wait(&sm.bar[QG_DQDONE + (n & 1)], (n >> 1) & 1, abort, 319) &&
                                   kfull(n + 2, 317)))
                            break;
                        tc_fence_after();
                        issue_s(n + 2);
                    }
                }
                // this thread's products complete before TMEM is released (after an abort too)
                mma_commit(&sm.bar[QG_SDONE]);
                if (!mbar_wait(&sm.bar[QG_SDONE], 0, abort, 322)) mbar_wait_drain(&sm.bar[QG_SDONE], 0);
            }
        }
    } else if (warp < 4) {
        reg_dealloc<56>();  // warp 3: idle
    } else {
        // ================================================ dS (thread = query row, 64 keys of each tile)
        const int hh = warp >= 8 ? 1 : 0, wq = warp & 3;
        if (hh == 0) reg_alloc<232>();
        else reg_alloc<216>();
        const int r = 32 * wq + lane, i = q0 + r;
        const bool valid = i < L.S;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        const int Spad = row_stride(L.S);
        const size_t rp = ((size_t)b * L.Hq + hq) * Spad + i;
        const int iq = valid ? i - L.q_off : 0;  // row of the query-side tensors (lse, q, dq)
        const size_t ro = ((size_t)b * L.Hq + hq) * L.Sq + iq;
        // the forward's log-sum-exp (base 2): its scores are these, bit for bit
        const float lse2 = valid ? p.P.lse[ro] * kLog2e : INFINITY;
        const float dai = valid ? p.dainv[rp] : 0.f;       // undoes the dA row scale
        float delta = valid ? p.P.delta[rp] : 0.f;         // sum_d dout out (gate pass)
        // largest ||v|| over the key tiles of the sweep (every lane of the warp takes a share)
        const size_t nst = (size_t)L.B * L.Hkv * nkt;
        const float* vstat = p.tstat + 2 * nst + ((size_t)b * L.Hkv + kvh) * nkt;
        float vmax = 0.f;
        for (int t = kt_lo + lane; t <= qb; t += 32) vmax = fmaxf(vmax, vstat[t]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
        // |dS_ij| = P |dP_ij - Delta_i| <= ||dA_i|| ||v_j|| + |Delta_i|, ||dA_i|| <= sqrt(D) max|dout_i|
        const float dmx = valid ? p.domax[rp] : 0.f;
        const float dsc = ldexpf(1.0f, fit_exp(sqrtf((float)kD) * dmx * vmax + fabsf(delta)));
        if (hh == 0 && i < Spad) {
            // per-row values of the key-major kernel's TMA loads; past S the neutral ones
            p.lse2p[rp] = lse2;
            if (!valid) {
                p.P.delta[rp] = 0.f;
                p.dainv[rp] = 0.f;
            }
        }
        const float* vtrow = p.vtinv + ((size_t)b * L.Hkv + kvh) * nkt;
        const int lo = max(i - L.W + 1, 0), hi = i;              // this row's visible keys
        const int rmin = q0 + 32 * wq, rmax = rmin + 31;        // rows of this warp
        float macc2[2] = {0.f, 0.f};                             // sum_j (dS_ij dsc) S_ij, two partials
        bool ok = true;
        for (int n = 0; n < N && ok; ++n) {
            const int kc0 = (kt_lo + n) * TF_BN + 64 * hh;       // first key of this half
            const float kd = dai * vtrow[kt_lo + n];             // dP = dv * kd on this tile
            if (!(ok = mbar_wait(&sm.bar[QG_SDPFULL], n & 1, abort, 320))) break;
            tc_fence_after();
            float sv[64], dv[64];
            const uint32_t ts = tm_s(n) + lane_off + 64 * hh;
            tmem_ld32f(ts, sv);
            tmem_ld32f(ts + 32, sv + 32);
            tmem_ld32f(TM_DP + lane_off + 64 * hh, dv);
            tmem_ld32f(TM_DP + lane_off + 64 * hh + 32, dv + 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar[QG_DPFREE]);
            // fully visible to the warp's rows unless the half crosses the diagonal or the
            // window's lower edge (warp-uniform)
            const bool full = kc0 + 63 <= rmin && kc0 > rmax - L.W;
            if (N == 1) {
                // Every row's window lies in this one tile: Delta = sum_j P dP from these very
                // products instead of the gate pass's sum_d dout out, whose bf16 `out` rounding
                // (2^-9) would leave dP - Delta short of cancelling where a row sees few keys
                // (a single key: dS = 0 exactly).  The key-major kernel reads it back.
                float part = 0.f;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const uint32_t vm = full ? 0xffffffffu : bit_range(lo - (kc0 + 32 * c), hi - (kc0 + 32 * c));
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float pv = fast_exp2(fmaf(sv[32 * c + e], c2, -lse2));
                        part = fmaf(((vm >> e) & 1u) ? pv : 0.f, dv[32 * c + e], part);
                    }
                }
                float* dpart = reinterpret_cast<float*>(sm.V[1][0]);
                dpart[hh * TF_BM + r] = part * kd;
                mbar_arrive(&sm.bar[QG_DELTA]);
                if (!(ok = mbar_wait(&sm.bar[QG_DELTA], 0, abort, 321))) break;
                delta = valid ? dpart[r] + dpart[TF_BM + r] : 0.f;
                if (hh == 0 && valid) p.P.delta[rp] = delta;
            }
            const float kds = kd * dsc, dls = delta * dsc;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t pk[16];
                if (full) {
                    qg_ds_chunk<false>(sv + 32 * c, dv + 32 * c, 0u, c2, lse2, kds, dls, macc2, pk);
                } else {
                    const uint32_t vm = bit_range(lo - (kc0 + 32 * c), hi - (kc0 + 32 * c));
                    qg_ds_chunk<true>(sv + 32 * c, dv + 32 * c, vm, c2, lse2, kds, dls, macc2, pk);
                }
                tmem_st16(tm_s(n) + lane_off + 64 * hh + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar[QG_DSFULL]);
        }
        // sum_j dS_ij S_ij (dsc, a power of two, divides out exactly)
        const float macc = (macc2[0] + macc2[1]) / dsc;
        if (hh == 1) {
            reinterpret_cast<float*>(sm.V[1][0])[256 + r] = macc;  // mdot_hi
            mbar_arrive(&sm.bar[QG_MDOT]);
        } else {
            // ------------------------------------------ dq epilogue: RoPE / RMSNorm backward
            const size_t off = ((size_t)(b * (size_t)L.Sq + iq) * L.Hq + hq) * kD;
            const float rinv = valid ? p.qrinv[((size_t)b * L.Hq + hq) * L.S + i] : 0.f;
            uint4 xv0[8];  // first half of the raw q row, in flight during the wait
#pragma unroll
            for (int c = 0; c < 8; ++c)
                xv0[c] = valid ? __ldg(reinterpret_cast<const uint4*>(L.q + off) + c) : make_uint4(0u, 0u, 0u, 0u);
            // d_gamma_q slices, one per warp, in the V ring (free once every product is done)
            float* dgam = reinterpret_cast<float*>(sm.V[0][0]) + wq * kD;
            if (ok && (ok = mbar_wait(&sm.bar[QG_DQFULL], 0, abort, 330) && mbar_wait(&sm.bar[QG_MDOT], 0, abort, 331))) {
                tc_fence_after();
                for (int d = lane; d < kD; d += 32) dgam[d] = 0.f;
                __syncwarp();
                float dy[128];
                tmem_ld32f(TM_DQ + lane_off, dy);
                tmem_ld32f(TM_DQ + lane_off + 32, dy + 32);
                tmem_ld32f(TM_DQ + lane_off + 64, dy + 64);
                tmem_ld32f(TM_DQ + lane_off + 96, dy + 96);
                tmem_wait_ld();
                const float f = L.scale / (dsc * oscale);
                const float mdot = (macc + reinterpret_cast<const float*>(sm.V[1][0])[256 + r]) * mdot_f;
                row_rope_rms_backward_regs<ANY ? 0 : TF_HALF>(dy, f, mdot, rinv, xv0, L.q + off, p.P.dq + off, valid, i,
                                                              sm.gq, dgam, L);
            }
        }
    }

    // ------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
    if (tid < kD) {
        const float* dg = reinterpret_cast<const float*>(sm.V[0][0]);
        p.P.dgq_part[(size_t)blockIdx.x * kD + tid] =
            sm.abort ? 0.f : (dg[tid] + dg[kD + tid]) + (dg[2 * kD + tid] + dg[3 * kD + tid]);
    }
    if (tid == 0 && sm.abort && p.err) atomicExch(p.err, sm.abort);
}

// The query-major kernel for windows wider than one tile: one CTA per unit, the instance for
// the layer's 21 rotated pairs or for any other number.
cudaError_t launch_bwd_q_glob(const BwdTcParams& p, int units, cudaStream_t stream) {
    auto k = p.P.L.rope_half != TF_HALF ? bwd_q_glob_kernel<true> : bwd_q_glob_kernel<false>;
    const size_t smem = bwd_q_glob_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<units, BQG_THREADS, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace zgcm
