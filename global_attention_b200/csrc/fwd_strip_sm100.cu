// fwd_strip_sm100.cu — gated sliding-window attention forward on tcgen05 / TMEM / TMA
// (sm_100a), organised by strips of positions.
//
// Layer (ZGCM-1; page citations in common.cuh): out = sigmoid(g) * softmax_window(q~ k~^T) v,
// q~, k~ the RMS-normalised (gamma) and partially rotated q, k; key j visible to query i iff
// i-W < j <= i.  This kernel takes windows W <= 128 (the 27 sliding layers use W = 128),
// 4 query heads per KV head (GQA 32/8) and any number of rotated dims.
//
// A strip is (batch b, KV head, 32 consecutive positions p0..p0+31) with the 4 query heads of
// the KV group: 128 query rows that share one window of keys, positions p0-128 .. p0+31 —
// five 32-key chunks.  The MMA tile's rows are (position, head) pairs, row = 4 pos + head (the
// order one TMA box {64 d, 4 heads, 32 positions} lands in), so one M=128 product covers the
// whole window of all 128 rows: no key tile is masked out entirely and every warp (8
// positions x 4 heads) sees the same mask shape.  The layer's 42 rotated dims take an unrolled
// prologue, other counts one that forms the angles where needed.  Consecutive strips of a
// chain share four of their five chunks; K and V chunks stream through an 8-slot ring, one
// new chunk per strip.
//
// Q~ and K~ are fp16 (times the power of two qk_fp16_scale picks), formed by the backward's own
// device function, angles and scale, so the scores equal the backward's bit for bit.  Two modes:
//   * plain forward: q and k arrive raw; K is normalised and rotated in the ring, in place, by
//     two converter warps (thread = key row) and Q by the prologue warpgroup: no scratch memory;
//   * the training pair (PREP): the preparation kernels have already formed Q~ and K~ (and every
//     row's inverse RMS) in the caller's activation store, which the backward reads; they arrive
//     by TMA ready to use and the converter and prologue warps stay idle.
// Per strip n (softmax warpgroup X = n mod 2, TMEM S_X):
//   S   = Q~ K~_span^T            tcgen05.mma M=128 N=160 K=128 (one or two runs of ring
//                                  slots, issued in turn), fp16 operands in smem
//   P   = exp2(S c - m)           softmax warpgroup X, thread = row, written as bf16 over the
//                                  front of S_X; m a bound on every score when small enough
//                                  (one pass), else the row maximum
//   O   = P V_span                tcgen05.mma M=128 N=128 K=160, P from TMEM, V MN-major
//   out = sigmoid(g) O / l        the same warpgroup, 16-byte loads and stores
// Two softmax warpgroups take alternate strips, so one's exponentials overlap the other's
// products and gate epilogue.  TMEM: S_0 [0,160), S_1 [160,320), O [320,448).  A strip that
// starts a new chain finishes the previous strip's P V before its own S (its five new chunks
// need the slots the previous strip holds).
//
// Warp roles (512 threads): w0 TMA producer (Q, K and V), w1 MMA issuer + TMEM owner, w2-3
// K converters (alternate chunks), w4-7 softmax/epilogue of even strips, w8-11 of odd strips,
// w12-15 Q prologue.  Every wait is bounded (and voted warp-uniform before warp-collective
// instructions); on expiry the CTA records the site, drains, frees TMEM and returns.
#include <cudaTypedefs.h>

#include "sm100.cuh"
#include "tc_rows.cuh"

namespace zgcm {
using namespace sm100;

namespace {

constexpr int SP = 32;                      // positions per strip
constexpr int SG = 4;                       // query heads per KV head
constexpr int SROWS = SP * SG;              // 128 MMA rows
constexpr int NCH = 5;                      // 32-key chunks in a strip's window span
constexpr int SPAN = NCH * 32;              // 160 keys: positions p0-128 .. p0+31
constexpr int RING = 8;                     // chunk slots of the K and V rings
constexpr uint32_t CHUNK_HALF = 32 * 128;   // one 32-row x 64-dim half of a chunk: 4 KB
constexpr uint32_t CHUNK_BYTES = 2 * CHUNK_HALF;
constexpr uint32_t QHALF = SROWS * 128;     // 16 KB
constexpr int THREADS = 512;
constexpr uint32_t TM_O = 2 * SPAN;         // O columns [320, 448)

struct StripParams {
    CUtensorMap tm_q;    // raw q bf16 {D, Hq, S, B}, box {64, 4, 32, 1}
    CUtensorMap tm_k;    // raw k bf16 {D, Hkv, S, B}, box {64, 1, 32, 1}
    CUtensorMap tm_v;    // raw v bf16, box {64, 1, 32, 1}
    LayerParams L;
    bf16* out;
    float* lse;
    int* err;
    int nst;             // strips per (b, KV head) chain: ceil(S / 32)
    int total;           // B * Hkv * nst
};

enum Bar {
    KF = 0,                 // [RING] raw K chunk landed
    VF = KF + RING,         // [RING] V chunk landed
    KC = VF + RING,         // [RING] K chunk converted
    KE = KC + RING,         // [RING] slot free (its last strip's products done)
    QF = KE + RING,         // [2] raw Q tile landed
    QR = QF + 2,            // [2] Q~ ready (prologue)
    QE = QR + 2,            // [2] Q buffer read by its S product
    SF = QE + 2,            // [2] S_X complete
    PF = SF + 2,            // [2] P_X written
    OF = PF + 2,            // [2] O complete for a strip of warpgroup X
    OE = OF + 2,            // [2] O read by warpgroup X's epilogue
    DONE = OE + 2,
    NBAR = DONE + 1
};

struct StripSmem {
    alignas(1024) unsigned char K[2][RING][CHUNK_HALF];   // [d-half][slot]: raw k -> K~ fp16
    alignas(1024) unsigned char V[2][RING][CHUNK_HALF];   // [d-half][slot]: v bf16
    alignas(1024) unsigned char Q[2][2][QHALF];           // [buffer][d-half]
    float2 cs[SP][TF_HALF];                               // (cos, sin) of the strip's positions
    float gq[kD], gk[kD];
    float mref;
    uint64_t bar[NBAR];
    uint32_t tmem_base;
    int abort;
};

struct Strip {
    int b, kvh, s;      // chain (b, KV head) and strip index in it (positions 32 s ..)
    bool fresh;         // first strip of a chain in this CTA: its whole span is loaded
};

__device__ __forceinline__ Strip strip_at(const StripParams& p, int t, int t_begin) {
    Strip st;
    const int chain = t / p.nst;
    st.s = t - chain * p.nst;
    st.b = chain / p.L.Hkv;
    st.kvh = chain - st.b * p.L.Hkv;
    st.fresh = (t == t_begin) || (st.s == 0);
    return st;
}

// S = Q~ K~_span^T over the span's ring slots: one run, or two around the ring's end, issued
// K-step by K-step in turn (independent accumulators, which the tensor pipe overlaps)
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc0, int s0, int run0) {
    const uint32_t id0 = idesc_f16(128, 32 * run0, false), id1 = idesc_f16(128, 32 * (NCH - run0), false);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t half = kk >> 2, within = (kk & 3) * 32;
        const uint32_t ao = half * QHALF + within, bo = half * RING * CHUNK_HALF + within;
        mma_ss(d_tmem, sdesc_step(q_desc, ao), sdesc_step(k_desc0, s0 * CHUNK_HALF + bo), id0, kk > 0 ? 1u : 0u);
        if (run0 < NCH)
            mma_ss(d_tmem + 32 * run0, sdesc_step(q_desc, ao), sdesc_step(k_desc0, bo), id1, kk > 0 ? 1u : 0u);
    }
}

}  // namespace

// PREP: Q~ and K~ (fp16) were formed by the preparation kernels into the activation store and
// arrive by TMA ready to use (the training pair, whose backward reads that store anyway): no
// prologue or converter work in this kernel.  Otherwise q and k arrive raw and are converted
// here.
// ANY: any number of rotated pairs (L.rope_half), the rotation angles formed where needed;
// otherwise the layer's 21 pairs, unrolled, with the angles of a strip shared by its heads.
template <bool PREP, bool ANY>
__global__ void __launch_bounds__(THREADS, 1) fwd_strip_kernel(const __grid_constant__ StripParams p) {
    const LayerParams& L = p.L;
    extern __shared__ unsigned char smem_raw[];
    StripSmem& sm = *reinterpret_cast<StripSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &sm.abort;
    const int t_begin = (int)(((long long)blockIdx.x * p.total) / gridDim.x);
    const int t_end = (int)(((long long)(blockIdx.x + 1) * p.total) / gridDim.x);
    const int nstrips = t_end - t_begin;

    if (tid == 0) {
        sm.abort = 0;
        for (int i = 0; i < RING; ++i) {
            mbar_init(&sm.bar[KF + i], 1);
            mbar_init(&sm.bar[VF + i], 1);
            mbar_init(&sm.bar[KC + i], 1);
            mbar_init(&sm.bar[KE + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.bar[QF + i], 1);
            mbar_init(&sm.bar[QR + i], 128);
            mbar_init(&sm.bar[QE + i], 1);
            mbar_init(&sm.bar[SF + i], 1);
            mbar_init(&sm.bar[PF + i], 128);
            mbar_init(&sm.bar[OF + i], 1);
            mbar_init(&sm.bar[OE + i], 128);
        }
        mbar_init(&sm.bar[DONE], 1);
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
    if (warp == 3) {
        // The exponentials' reference: a bound on every score (an RMS-normalised row has norm
        // at most sqrt(D) before gamma and the rotation keeps norms), used when at most 60.
        float amax_q = 0.f, amax_k = 0.f;
        for (int d = lane; d < kD; d += 32) {
            amax_q = fmaxf(amax_q, fabsf(L.gamma_q[d]));
            amax_k = fmaxf(amax_k, fabsf(L.gamma_k[d]));
        }
        for (int o = 16; o > 0; o >>= 1) {
            amax_q = fmaxf(amax_q, __shfl_xor_sync(0xffffffffu, amax_q, o));
            amax_k = fmaxf(amax_k, __shfl_xor_sync(0xffffffffu, amax_k, o));
        }
        if (lane == 0) sm.mref = fabsf(L.scale_log2) * (float)kD * amax_q * amax_k * 1.001f + 0.25f;
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k);
        prefetch_tmap(&p.tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    const float c2 = L.scale_log2 / (oscale * oscale);  // S holds oscale^2 q~.k~

    if (warp == 0) {
        // ================================================ TMA producer: Q tiles and K/V chunks
        // Both streams run ahead independently, each bounded by its buffers; the thread polls
        // whichever can move (a blocking wait on one could stall the other).
        if (lane == 0) {
            int nq = 0, tq = t_begin;        // next Q tile (strip)
            int lk = 0, tk = t_begin, ck = 0, nck = 0;  // next load, its strip, chunk, loads left of it
            Strip stk{};
            int last_q[2] = {-1, -1}, last_l[RING];
            for (int i = 0; i < RING; ++i) last_l[i] = -1;
            uint32_t idle = 0;
            while ((nq < nstrips || tk < t_end) && !*abort) {
                bool moved = false;
                if (nq < nstrips) {
                    const int buf = nq & 1;
                    const uint32_t ph = ((nq >> 1) - 1) & 1;
                    if (nq < 2 || mbar_try_wait(&sm.bar[QE + buf], ph)) {
                        const Strip st = strip_at(p, tq, t_begin);
                        mbar_expect_tx(&sm.bar[QF + buf], 2 * QHALF);
                        tma_load_4d(sm.Q[buf][0], &p.tm_q, &sm.bar[QF + buf], 0, st.kvh * SG, st.s * SP, st.b);
                        tma_load_4d(sm.Q[buf][1], &p.tm_q, &sm.bar[QF + buf], 64, st.kvh * SG, st.s * SP, st.b);
                        last_q[buf] = nq;
                        ++nq;
                        ++tq;
                        moved = true;
                    }
                }
                if (tk < t_end) {
                    if (nck == 0) {  // the loads of strip tk: its whole span when fresh, else one chunk
                        stk = strip_at(p, tk, t_begin);
                        nck = stk.fresh ? NCH : 1;
                        ck = stk.s - nck + 1;
                    }
                    const int slot = lk % RING;
                    if (lk < RING || mbar_try_wait(&sm.bar[KE + slot], ((lk / RING) - 1) & 1)) {
                        mbar_expect_tx(&sm.bar[KF + slot], CHUNK_BYTES);
                        tma_load_4d(sm.K[0][slot], &p.tm_k, &sm.bar[KF + slot], 0, stk.kvh, ck * 32, stk.b);
                        tma_load_4d(sm.K[1][slot], &p.tm_k, &sm.bar[KF + slot], 64, stk.kvh, ck * 32, stk.b);
                        mbar_expect_tx(&sm.bar[VF + slot], CHUNK_BYTES);
                        tma_load_4d(sm.V[0][slot], &p.tm_v, &sm.bar[VF + slot], 0, stk.kvh, ck * 32, stk.b);
                        tma_load_4d(sm.V[1][slot], &p.tm_v, &sm.bar[VF + slot], 64, stk.kvh, ck * 32, stk.b);
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
                    *abort = 1;
                    break;
                }
            }
            // every copy issued must have landed before the CTA exits (matters after an abort)
            for (int b = 0; b < 2; ++b)
                if (last_q[b] >= 0) mbar_wait_drain(&sm.bar[QF + b], (last_q[b] >> 1) & 1);
            for (int sl = 0; sl < RING; ++sl)
                if (last_l[sl] >= 0) {
                    mbar_wait_drain(&sm.bar[KF + sl], (last_l[sl] / RING) & 1);
                    mbar_wait_drain(&sm.bar[VF + sl], (last_l[sl] / RING) & 1);
                }
        }
    } else if (warp == 1) {
        // ================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_O = idesc_bf16(128, 128, true);
            const uint64_t q_desc0 = sdesc_sw128(smem_u32(sm.Q[0][0]), 16, 1024);
            const uint64_t k_desc0 = sdesc_sw128(smem_u32(sm.K[0][0]), 16, 1024);
            const uint64_t v_desc0 = sdesc_sw128(smem_u32(sm.V[0][0]), RING * CHUNK_HALF, 1024);
            int kc_waited = 0, vf_waited = 0;
            int lend[2] = {0, 0};   // newest load of the strips in flight, by parity
            bool ok = true;
            auto issue_pv = [&](int m, bool last) -> bool {
                const int X = m & 1;
                if (!mbar_wait(&sm.bar[PF + X], (m >> 1) & 1, abort, 40)) return false;
                const int le = lend[X];
                for (; vf_waited <= le; ++vf_waited)
                    if (!mbar_wait(&sm.bar[VF + vf_waited % RING], (vf_waited / RING) & 1, abort, 41)) return false;
                if (m >= 1 && !mbar_wait(&sm.bar[OE + ((m - 1) & 1)], ((m - 1) >> 1) & 1, abort, 42)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 2 * NCH; ++kk) {
                    const int slot = (le - (NCH - 1) + (kk >> 1)) % RING;
                    const uint64_t bdesc = sdesc_step(v_desc0, slot * CHUNK_HALF + (kk & 1) * 2048);
                    mma_ts(tmem + TM_O, tmem + X * SPAN + kk * 8, bdesc, IDESC_O, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar[OF + X]);
                // release the chunks no later strip reads: all of them before a fresh strip or at
                // the end, else the oldest
                const int keep_from = last ? le + 1 : lend[X ^ 1] - (NCH - 1);
                for (int l = le - (NCH - 1); l <= le && l < keep_from; ++l) mma_commit(&sm.bar[KE + l % RING]);
                return true;
            };
            int lcount = 0;
            for (int n = 0; n < nstrips && ok; ++n) {
                const Strip st = strip_at(p, t_begin + n, t_begin);
                lcount += st.fresh ? NCH : 1;
                const int le = lcount - 1, X = n & 1, buf = n & 1;
                lend[X] = le;
                // A fresh strip (a new chain) needs five new chunks while the previous strip still
                // holds five of the eight slots: finish the previous strip first, which frees them.
                // Otherwise S(n) goes first, so this strip's softmax overlaps the previous P V.
                const bool pv_first = st.fresh && n >= 1;
                if (pv_first && !(ok = issue_pv(n - 1, false))) break;
                if (!(ok = mbar_wait(&sm.bar[(PREP ? QF : QR) + buf], (n >> 1) & 1, abort, 43))) break;
                for (; kc_waited <= le && ok; ++kc_waited)
                    ok = mbar_wait(&sm.bar[(PREP ? KF : KC) + kc_waited % RING], (kc_waited / RING) & 1, abort, 44);
                if (!ok) break;
                tc_fence_after();
                // S = Q~ K~_span^T: the span's slots le-4 .. le, in one run or two around the ring end
                const int s0 = (le - (NCH - 1)) % RING;
                const int run0 = min(NCH, RING - s0);
                issue_s(tmem + X * SPAN, sdesc_step(q_desc0, buf * 2 * QHALF), k_desc0, s0, run0);
                mma_commit(&sm.bar[QE + buf]);
                mma_commit(&sm.bar[SF + X]);
                if (n >= 1 && !pv_first) ok = issue_pv(n - 1, false);
            }
            if (ok && nstrips > 0) issue_pv(nstrips - 1, true);
            // every MMA issued must complete before TMEM is released
            mma_commit(&sm.bar[DONE]);
            mbar_wait_drain(&sm.bar[DONE], 0);
        }
    } else if ((warp == 2 || warp == 3) && !PREP) {
        // ================================================ K converters: normalise + rotate in place
        // warp 2 takes the even loads, warp 3 the odd ones; thread = key row of the chunk
        const int mine = warp - 2;
        int l = 0;
        bool ok = true;
        for (int t = t_begin; t < t_end && ok; ++t) {
            const Strip st = strip_at(p, t, t_begin);
            const int nl = st.fresh ? NCH : 1;
            for (int c = 0; c < nl && ok; ++c, ++l) {
                if ((l & 1) != mine) continue;
                const int chunk = st.s - nl + 1 + c, slot = l % RING;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar[KF + slot], (l / RING) & 1, abort, 50)))) break;
                const int pos = chunk * 32 + lane;
                if constexpr (ANY)
                    tf_prologue_row_any<true>(sm.K[0][slot], sm.K[1][slot], lane, sm.gk, L, pos, oscale);
                else
                    tf_prologue_row_at<true>(sm.K[0][slot], sm.K[1][slot], lane, sm.gk, L,
                                             [&](int q) {
                                                 float2 w;
                                                 rope_cs(L.theta[q], pos, w.x, w.y);
                                                 return w;
                                             },
                                             oscale);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.bar[KC + slot]);
            }
        }
    } else if (warp >= 12 && !PREP) {
        // ================================================ Q prologue: Q~ normalised + rotated in place
        const int m = tid - 384, pos = m >> 2;
        bool ok = true;
        for (int n = 0; n < nstrips && ok; ++n) {
            const Strip st = strip_at(p, t_begin + n, t_begin);
            const int p0 = st.s * SP, buf = n & 1;
            // angles of the strip's positions: the 4 threads of a position (its 4 heads, all in this
            // warp) take pairs t = head, head + 4, ..; only this warp reads its 8 positions' entries
            __syncwarp();   // the previous strip's rows have read the table
            for (int q = m & 3; !ANY && q < TF_HALF; q += 4) {
                float2 w;
                rope_cs(L.theta[q], p0 + pos, w.x, w.y);
                sm.cs[pos][q] = w;
            }
            __syncwarp();
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar[QF + buf], (n >> 1) & 1, abort, 60)))) break;
            if constexpr (ANY)
                tf_prologue_row_any<true>(sm.Q[buf][0], sm.Q[buf][1], m, sm.gq, L, p0 + pos, oscale);
            else
                tf_prologue_row_at<true>(sm.Q[buf][0], sm.Q[buf][1], m, sm.gq, L, [&](int q) { return sm.cs[pos][q]; },
                                         oscale);
            fence_proxy_async_smem();
            mbar_arrive(&sm.bar[QR + buf]);
        }
    } else if (warp >= 4 && warp < 12) {
        // ================================================ softmax + gate epilogue (thread = row)
        const int X = (warp - 4) >> 2;           // 0: even strips, 1: odd strips
        const int m = tid - 128 * (1 + X);       // row of the tile: 4 * position + head
        const int pos = m >> 2;
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t TS = tmem + X * SPAN;
        for (int n = X; n < nstrips; n += 2) {
            const Strip st = strip_at(p, t_begin + n, t_begin);
            const int p0 = st.s * SP, i = p0 + pos, h = st.kvh * SG + (m & 3);
            const bool valid = i < L.S;
            // visible span offsets o (key = p0 - 128 + o): i - W < key <= i, key >= 0
            const int olo = max(max(pos + 129 - L.W, 128 - p0), 0), ohi = pos + 128;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar[SF + X], (n >> 1) & 1, abort, 70))) break;
            tc_fence_after();
            float mu = sm.mref;
            if (!(mu <= 60.f)) {
                float mx = -INFINITY;
#pragma unroll 1
                for (int c = 0; c < NCH; ++c) {
                    const uint32_t vm = bit_range(olo - 32 * c, ohi - 32 * c);
                    if (__all_sync(0xffffffffu, vm == 0u)) continue;
                    float v[32];
                    tmem_ld32f(TS + lane_off + 32 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) mx = fmaxf(mx, ((vm >> e) & 1u) ? v[e] : -INFINITY);
                }
                mu = (mx == -INFINITY) ? 0.f : mx * c2;
            }
            float l = 0.f;
#pragma unroll 1
            for (int c = 0; c < NCH; ++c) {
                const uint32_t vm = bit_range(olo - 32 * c, ohi - 32 * c);
                uint32_t pk[16];
                if (__all_sync(0xffffffffu, vm == 0xffffffffu)) {
                    // every key visible to the warp's rows: no mask, scores two at a time
                    float v[32];
                    tmem_ld32f(TS + lane_off + 32 * c, v);
                    tmem_wait_ld();
                    const float2 cc = make_float2(c2, c2), nm = make_float2(-mu, -mu);
                    float2 la = make_float2(0.f, 0.f), lb = la;
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        const float2 xa = ffma2(make_float2(v[e], v[e + 1]), cc, nm);
                        const float2 xb = ffma2(make_float2(v[e + 2], v[e + 3]), cc, nm);
                        const float2 pa = make_float2(fast_exp2(xa.x), fast_exp2(xa.y));
                        const float2 pb = make_float2(fast_exp2(xb.x), fast_exp2(xb.y));
                        la = fadd2(la, pa);
                        lb = fadd2(lb, pb);
                        pk[e >> 1] = pack_bf16(pa.x, pa.y);
                        pk[(e >> 1) + 1] = pack_bf16(pb.x, pb.y);
                    }
                    la = fadd2(la, lb);
                    l += la.x + la.y;
                } else if (!__all_sync(0xffffffffu, vm == 0u)) {
                    float v[32];
                    tmem_ld32f(TS + lane_off + 32 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float p0v = fast_exp2(v[e] * c2 - mu), p1v = fast_exp2(v[e + 1] * c2 - mu);
                        p0v = ((vm >> e) & 1u) ? p0v : 0.f;  // (a masked score may overflow: selected away)
                        p1v = ((vm >> (e + 1)) & 1u) ? p1v : 0.f;
                        l += p0v + p1v;
                        pk[e >> 1] = pack_bf16(p0v, p1v);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                }
                tmem_st16(TS + lane_off + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar[PF + X]);
            if (valid) p.lse[((size_t)st.b * L.Hq + h) * L.S + i] = (mu + __log2f(l)) * kLn2;
            // gate epilogue: out = sigmoid(g) * O / l
            const size_t off = ((size_t)(st.b * (size_t)L.S + (valid ? i : 0)) * L.Hq + h) * kD;
            uint4 gr[16];
            if (valid) {
#pragma unroll
                for (int c = 0; c < 16; ++c) gr[c] = __ldg(reinterpret_cast<const uint4*>(L.g + off) + c);
            }
            const float hi = 0.5f / l;
            const float2 hinv = make_float2(hi, hi);
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar[OF + X], (n >> 1) & 1, abort, 71))) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + TM_O + lane_off + 32 * c, v);
                tmem_wait_ld();
                if (c == 3) {
                    tc_fence_before();
                    mbar_arrive(&sm.bar[OE + X]);
                }
                if (valid) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const uint4 g4 = gr[4 * c + q4];
                        const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
                        uint32_t ow[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            // sigmoid(x) / l = (0.5 + 0.5 tanh(x / 2)) / l, two columns at a time
                            const float2 hg = fmul2(unpack_bf16(gw[e2]), make_float2(0.5f, 0.5f));
                            const float2 th = make_float2(fast_tanh(hg.x), fast_tanh(hg.y));
                            const float2 sg = ffma2(th, hinv, hinv);
                            const int col = 8 * q4 + 2 * e2;
                            const float2 o = fmul2(make_float2(__uint_as_float(v[col]), __uint_as_float(v[col + 1])), sg);
                            ow[e2] = pack_bf16(o.x, o.y);
                        }
                        *reinterpret_cast<uint4*>(p.out + off + 32 * c + 8 * q4) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
            }
        }
    }

    // ------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
    if (tid == 0 && sm.abort && p.err) atomicExch(p.err, sm.abort);
}

// ------------------------------------------------------------------ host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 strip_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 4-D 16-bit map {D, H, S, B} (innermost first), box {64, heads, rows, 1}, 128-byte swizzle
bool strip_map(CUtensorMap* map, const void* base, int H, int S, int B, CUtensorMapDataType dtype, int heads,
               int rows) {
    auto enc = strip_encoder();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)S * H * kD * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)heads, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Windows up to 128 keys, 4 query heads per KV head (any number of rotated dims).
bool fwd_strip_supported(const LayerParams& L) {
    return L.W <= 128 && L.G == SG && L.S >= 1 && L.B >= 1;
}

namespace {
template <bool PREP>
cudaError_t launch_strip_kernel(const StripParams& p, int grid, size_t smem, cudaStream_t stream) {
    auto k = p.L.rope_half == TF_HALF ? fwd_strip_kernel<PREP, false> : fwd_strip_kernel<PREP, true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, THREADS, smem, stream>>>(p);
    return cudaGetLastError();
}
}  // namespace

size_t fwd_strip_smem_bytes() { return sizeof(StripSmem) + 1024; }

cudaError_t launch_fwd_prep_k(const LayerParams& L, void* workspace, int* err_word, cudaStream_t stream,
                              float* krinv);
cudaError_t launch_prep_q_only(const LayerParams& L, void* q16, float* qrinv, int* err_word, cudaStream_t stream);

// The strip forward.  With `sv` (the training pair) the preparation kernels first form Q~, K~
// (fp16) and every q and k row's inverse RMS in the caller's activation store, which the
// backward reads, and the attention kernel loads Q~ and K~ from there; without it the kernel
// converts q and k itself and uses no scratch memory.
cudaError_t launch_fwd_strip(const FwdParams& fp, int* err_word, cudaStream_t stream, const SavedAct* sv) {
    StripParams p;
    p.L = fp.L;
    p.out = fp.out;
    p.lse = fp.lse;
    p.err = err_word;
    const LayerParams& L = fp.L;
    p.nst = (L.S + SP - 1) / SP;
    const long long total = (long long)L.B * L.Hkv * p.nst;
    if (total > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.total = (int)total;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const size_t smem = fwd_strip_smem_bytes();
    const int grid = (int)(total < sms ? total : sms);
    if (!strip_map(&p.tm_v, L.v, L.Hkv, L.S, L.B, BF, 1, 32)) return cudaErrorInvalidValue;
    if (sv) {
        // the training pair: Q~ and K~ (and the rows' inverse RMS) into the store first, then the
        // attention kernel reads them from there
        if ((e = launch_fwd_prep_k(L, sv->k16, err_word, stream, sv->krinv)) != cudaSuccess) return e;
        if ((e = launch_prep_q_only(L, sv->q16, sv->qrinv, err_word, stream)) != cudaSuccess) return e;
        if (!strip_map(&p.tm_q, sv->q16, L.Hq, L.S, L.B, F16, SG, SP) ||
            !strip_map(&p.tm_k, sv->k16, L.Hkv, L.S, L.B, F16, 1, 32))
            return cudaErrorInvalidValue;
        return launch_strip_kernel<true>(p, grid, smem, stream);
    }
    if (!strip_map(&p.tm_q, L.q, L.Hq, L.S, L.B, BF, SG, SP) || !strip_map(&p.tm_k, L.k, L.Hkv, L.S, L.B, BF, 1, 32))
        return cudaErrorInvalidValue;
    return launch_strip_kernel<false>(p, grid, smem, stream);
}

}  // namespace zgcm
