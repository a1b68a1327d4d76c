// fwd_sm100.cu — gated sliding-window attention forward on tcgen05 / TMEM / TMA (sm_100a).
//
// Layer (ZGCM-1; page citations in common.cuh): out = sigmoid(g) * softmax_window(q~ k~^T) v,
// with q~, k~ the RMS-normalised (gamma) and partially rotated q, k, window i-W < j <= i.
// This kernel takes windows W <= 128 (the 27 sliding layers use W = 128) and any number of
// query heads per KV head (the strip kernel, fwd_strip_sm100.cu, takes the layer's 4).
//
// Work decomposition: a "step" is (batch b, KV head, 128-query block qb) with all Hq/Hkv
// query heads of the group.  With W <= 128 the window of block qb lies inside key tiles
// qb-1 and qb, so consecutive steps of one (b, KV head) chain share a tile: a persistent
// CTA sweeps a contiguous range of steps and loads ONE new K/V tile per step into a 2-slot
// ring.  K~ (fp16, normalised and rotated once per tile by fwd_prep_k_kernel into the
// workspace) arrives by TMA ready to use; Q~ is normalised/rotated in place in shared memory
// (TMA-loaded raw, 128-byte swizzle = the UMMA K-major canonical layout).  Both are fp16
// times a power of two (qk_fp16_scale) that keeps them in range.
//
// Per head m (TMEM: S/P columns [0,256), O double buffer [256,384) and [384,512)):
//   S   = Q~ [K~_slot0; K~_slot1]^T          tcgen05.mma M=128 N=256 K=128, A,B in smem
//                                            (fp16 q~, k~, the backward's operands, so the
//                                            backward recomputes these scores bit for bit)
//   P   = exp2(S*scale*log2e - m)            softmax warpgroup, thread = query row, fp32,
//                                            written back as bf16 over the front of S; m is
//                                            a bound on every score of the launch when that
//                                            is small enough (one pass), else the row max
//   O   = P [V_slot0; V_slot1]               tcgen05.mma M=128 N=128 K=256, A in TMEM,
//                                            B (V, d-contiguous) MN-major in smem
//   out = sigmoid(g) * O / l                 epilogue, 16-byte global loads/stores
//
// Warp roles (512 threads): w0 TMA K/V, w1 MMA issue + TMEM owner, w2 TMA Q, w3 idle,
// w4-7 softmax, w8-11 prologue (Q~ in place; with save_q it also stores Q~ and the rows'
// inverse RMS for the backward), w12-15 gate epilogue.  Every wait is bounded; on expiry
// the CTA records the site, drains, frees TMEM and returns.
#include <cudaTypedefs.h>

#include "sm100.cuh"
#include "tc_rows.cuh"

namespace zgcm {
using namespace sm100;

constexpr int TF_THREADS = 512;

struct FwdTcParams {
    CUtensorMap tm_q;   // {D, Hq, S, B}, box {64, 1, 128, 1}, 128B swizzle
    CUtensorMap tm_k16; // K~ fp16 {D, Hkv, S, B} (fwd_prep_k_kernel, in the workspace)
    CUtensorMap tm_v;
    CUtensorMap tm_q16s; // Q~ fp16 {D, Hq, S, B} kept for the backward, box {64, 1, 32, 1} (save_q)
    LayerParams L;
    bf16* out;
    float* lse;
    float* qrinv;       // inverse RMS of each q row, [B,Hq,S] (save_q)
    int* err;           // device error word: site of an expired wait (0 = none)
    int total_steps;    // B * Hkv * ceil(S / 128)
    int save_q;         // keep Q~ and the q rows' inverse RMS for the backward
};

enum Bar {
    B_KFULL = 0, B_KEMPTY = 2, B_VFULL = 4, B_VEMPTY = 6,
    B_QFULL = 8, B_QREADY = 10, B_QEMPTY = 12,
    B_SFULL = 14, B_PFULL = 15,
    B_OFULL = 16, B_OEMPTY = 18, B_LFULL = 20, B_LEMPTY = 22,
    B_DONE = 24,
    B_QSTORED = 25,  // a Q buffer's rows were read by the stores that keep Q~ (save_q), by buffer
    B_COUNT = 27
};

struct FwdTcSmem {
    // ring of two K (resp. V) tiles, split by d-half so the 256 rows of a half are
    // contiguous: K[h] holds rows slot0(0..127), slot1(128..255) of dims 64h..64h+63
    alignas(1024) unsigned char K[2][TF_RING_HALF];
    alignas(1024) unsigned char V[2][TF_RING_HALF];
    alignas(1024) unsigned char Q[2][2][TF_HALF_BYTES];  // [buffer][d-half]
    float2 cs[TF_HALF][TF_BM];   // (cos, sin) of pair t at row r's position; thread r's column
    float gq[kD], gk[kD];
    float rowinv[2][TF_BM];
    float mref;   // bound on |scores| in exp2 units: the softmax's reference when small enough
    uint64_t bar[B_COUNT];
    uint32_t tmem_base;
    int abort;
};

// ------------------------------------------------------------------ the kernel

// ANY: any number of rotated pairs (L.rope_half), the angles formed per row as needed.
template <bool ANY>
__global__ void __launch_bounds__(TF_THREADS, 1) fwd_tc_kernel(const __grid_constant__ FwdTcParams p) {
    const LayerParams& L = p.L;
    extern __shared__ unsigned char smem_raw[];
    FwdTcSmem& sm = *reinterpret_cast<FwdTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &sm.abort;

    const int G = L.G;
    const int t_begin = (int)(((long long)blockIdx.x * p.total_steps) / gridDim.x);
    const int t_end = (int)(((long long)(blockIdx.x + 1) * p.total_steps) / gridDim.x);

    if (tid == 0) {
        sm.abort = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.bar[B_KFULL + i], 1);
            mbar_init(&sm.bar[B_KEMPTY + i], 1);
            mbar_init(&sm.bar[B_VFULL + i], 1);
            mbar_init(&sm.bar[B_VEMPTY + i], 1);
            mbar_init(&sm.bar[B_QFULL + i], 1);
            mbar_init(&sm.bar[B_QREADY + i], 128);
            mbar_init(&sm.bar[B_QEMPTY + i], 1);
            mbar_init(&sm.bar[B_OFULL + i], 1);
            mbar_init(&sm.bar[B_OEMPTY + i], 128);
            mbar_init(&sm.bar[B_LFULL + i], 128);
            mbar_init(&sm.bar[B_LEMPTY + i], 128);
        }
        mbar_init(&sm.bar[B_SFULL], 1);
        mbar_init(&sm.bar[B_PFULL], 128);
        mbar_init(&sm.bar[B_DONE], 1);
        for (int i = 0; i < 2; ++i) mbar_init(&sm.bar[B_QSTORED + i], 4);  // lane 0 of each prologue warp
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
        // Reference of the exponentials: a bound on every score rather than each row's maximum,
        // which saves a pass over the scores.  An RMS-normalised row has norm at most sqrt(D)
        // before gamma, and the rotation keeps norms, so |q~.k~| <= D max|gamma_q| max|gamma_k|;
        // with that as the reference no weight exceeds 1 and none falls below 2^(-2 mref).  Where
        // the bound is above 60 (far from fp32 / bf16 underflow) the rows take their maximum.
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
        prefetch_tmap(&p.tm_k16);
        prefetch_tmap(&p.tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t TM_S = tmem, TM_P = tmem, TM_O0 = tmem + 256;
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    const float c2 = L.scale_log2 / (oscale * oscale);  // S holds oscale^2 q~.k~

    if (warp == 0) {
        // ================================================ K / V producer
        if (lane == 0) {
            int n_next = 0;
            int last_k[2] = {-1, -1}, last_v[2] = {-1, -1};  // last tile issued per slot
            auto load_tile = [&](int n, int b, int kvh, int kt) -> bool {
                const int slot = n & 1;
                if (n >= 2 && !mbar_wait(&sm.bar[B_KEMPTY + slot], ((n >> 1) - 1) & 1, abort, 1)) return false;
                mbar_expect_tx(&sm.bar[B_KFULL + slot], TF_TILE_BYTES);
                tma_load_4d(sm.K[0] + slot * TF_HALF_BYTES, &p.tm_k16, &sm.bar[B_KFULL + slot], 0, kvh, kt * TF_BN, b);
                tma_load_4d(sm.K[1] + slot * TF_HALF_BYTES, &p.tm_k16, &sm.bar[B_KFULL + slot], 64, kvh, kt * TF_BN, b);
                last_k[slot] = n;
                if (n >= 2 && !mbar_wait(&sm.bar[B_VEMPTY + slot], ((n >> 1) - 1) & 1, abort, 2)) return false;
                mbar_expect_tx(&sm.bar[B_VFULL + slot], TF_TILE_BYTES);
                tma_load_4d(sm.V[0] + slot * TF_HALF_BYTES, &p.tm_v, &sm.bar[B_VFULL + slot], 0, kvh, kt * TF_BN, b);
                tma_load_4d(sm.V[1] + slot * TF_HALF_BYTES, &p.tm_v, &sm.bar[B_VFULL + slot], 64, kvh, kt * TF_BN, b);
                last_v[slot] = n;
                return true;
            };
            for (int t = t_begin; t < t_end && !*abort; ++t) {
                const StepInfo st = decode_step(L, t, t_begin, t_end);
                if (st.fresh && !load_tile(n_next++, st.b, st.kvh, st.qb - 1)) break;
                if (!load_tile(n_next++, st.b, st.kvh, st.qb)) break;
            }
            // every copy issued must have landed before the CTA exits (matters after an abort)
            for (int slot = 0; slot < 2; ++slot) {
                if (last_k[slot] >= 0) mbar_wait_drain(&sm.bar[B_KFULL + slot], (last_k[slot] >> 1) & 1);
                if (last_v[slot] >= 0) mbar_wait_drain(&sm.bar[B_VFULL + slot], (last_v[slot] >> 1) & 1);
            }
        }
    } else if (warp == 2) {
        // ================================================ Q producer
        if (lane == 0) {
            int m = 0;
            int last_q[2] = {-1, -1};
            for (int t = t_begin; t < t_end && !*abort; ++t) {
                const StepInfo st = decode_step(L, t, t_begin, t_end);
                for (int h = 0; h < G; ++h, ++m) {
                    const int buf = m & 1;
                    if (m >= 2 && !mbar_wait(&sm.bar[B_QEMPTY + buf], ((m >> 1) - 1) & 1, abort, 3)) break;
                    if (p.save_q && m >= 2 && !mbar_wait(&sm.bar[B_QSTORED + buf], ((m >> 1) - 1) & 1, abort, 4))
                        break;
                    mbar_expect_tx(&sm.bar[B_QFULL + buf], TF_TILE_BYTES);
                    const int hg = st.kvh * G + h;
                    tma_load_4d(sm.Q[buf][0], &p.tm_q, &sm.bar[B_QFULL + buf], 0, hg, st.qb * TF_BM, st.b);
                    tma_load_4d(sm.Q[buf][1], &p.tm_q, &sm.bar[B_QFULL + buf], 64, hg, st.qb * TF_BM, st.b);
                    last_q[buf] = m;
                }
            }
            for (int buf = 0; buf < 2; ++buf)
                if (last_q[buf] >= 0) mbar_wait_drain(&sm.bar[B_QFULL + buf], (last_q[buf] >> 1) & 1);
        }
    } else if (warp == 1) {
        // ================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_f16(128, 256, false);
            constexpr uint32_t IDESC_O = idesc_bf16(128, 128, true);
            const uint32_t q_base = smem_u32(sm.Q[0][0]);
            // descriptors of each operand's first 16-element step; the others are offsets
            const uint64_t q_desc0 = sdesc_sw128(q_base, 16, 1024);
            const uint64_t k_desc0 = sdesc_sw128(smem_u32(sm.K[0]), 16, 1024);
            const uint64_t v_desc0 = sdesc_sw128(smem_u32(sm.V[0]), TF_RING_HALF, 1024);
            int n_next = 0, n_prev = 0, n_cur = 0, m = 0;
            bool ok = true;
            for (int t = t_begin; t < t_end && ok; ++t) {
                const StepInfo st = decode_step(L, t, t_begin, t_end);
                if (st.fresh) {
                    n_prev = n_next++;
                    n_cur = n_next++;
                    ok = mbar_wait(&sm.bar[B_KFULL + (n_prev & 1)], (n_prev >> 1) & 1, abort, 10) &&
                         mbar_wait(&sm.bar[B_VFULL + (n_prev & 1)], (n_prev >> 1) & 1, abort, 11);
                } else {
                    n_prev = n_cur;
                    n_cur = n_next++;
                }
                ok = ok && mbar_wait(&sm.bar[B_KFULL + (n_cur & 1)], (n_cur >> 1) & 1, abort, 12) &&
                     mbar_wait(&sm.bar[B_VFULL + (n_cur & 1)], (n_cur >> 1) & 1, abort, 13);
                for (int h = 0; h < G && ok; ++h, ++m) {
                    const int buf = m & 1;
                    if (!(ok = mbar_wait(&sm.bar[B_QREADY + buf], (m >> 1) & 1, abort, 14))) break;
                    tc_fence_after();
                    // S = Q~ K~^T over both ring slots (N = 256), K = 128 in 8 steps of 16
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t half = kk >> 2, within = (kk & 3) * 32;
                        const uint64_t a = sdesc_step(q_desc0, buf * 2 * TF_HALF_BYTES + half * TF_HALF_BYTES + within);
                        const uint64_t bdesc = sdesc_step(k_desc0, half * TF_RING_HALF + within);
                        mma_ss(TM_S, a, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sm.bar[B_QEMPTY + buf]);
                    mma_commit(&sm.bar[B_SFULL]);
                    if (h == G - 1) {
                        mma_commit(&sm.bar[B_KEMPTY + (n_prev & 1)]);
                        if (st.release_cur) mma_commit(&sm.bar[B_KEMPTY + (n_cur & 1)]);
                    }
                    if (!(ok = mbar_wait(&sm.bar[B_PFULL], m & 1, abort, 15))) break;
                    if (m >= 2 && !(ok = mbar_wait(&sm.bar[B_OEMPTY + buf], ((m >> 1) - 1) & 1, abort, 16))) break;
                    tc_fence_after();
                    // O = P V: P bf16 in TMEM (16 keys = 8 columns per step), V MN-major
#pragma unroll
                    for (int kk = 0; kk < 16; ++kk) {
                        const uint64_t bdesc = sdesc_step(v_desc0, kk * 16 * 128);
                        mma_ts(TM_O0 + buf * 128, TM_P + kk * 8, bdesc, IDESC_O, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sm.bar[B_OFULL + buf]);
                    if (h == G - 1) {
                        mma_commit(&sm.bar[B_VEMPTY + (n_prev & 1)]);
                        if (st.release_cur) mma_commit(&sm.bar[B_VEMPTY + (n_cur & 1)]);
                    }
                }
            }
            // every MMA issued must complete before TMEM is released
            mma_commit(&sm.bar[B_DONE]);
            mbar_wait(&sm.bar[B_DONE], 0, abort, 17);
        }
    } else if (warp >= 4 && warp < 8) {
        // ================================================ softmax (thread = query row)
        const int r = tid - 128, wq = warp - 4;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        int n_next = 0, n_prev = 0, n_cur = 0, m = 0;
        for (int t = t_begin; t < t_end; ++t) {
            const StepInfo st = decode_step(L, t, t_begin, t_end);
            if (st.fresh) { n_prev = n_next++; n_cur = n_next++; } else { n_prev = n_cur; n_cur = n_next++; }
            const int q0 = st.qb * TF_BM, i = q0 + r;
            // key position of ring column c: slot (c >> 7) holds tile qb (cur) or qb-1 (prev)
            const int slot_cur = n_cur & 1;
            const int base0 = (slot_cur == 0 ? q0 : q0 - TF_BN), base1 = (slot_cur == 1 ? q0 : q0 - TF_BN);
            const int imin = q0 + 32 * wq, imax = imin + 31;
            bool stop = false;
            for (int h = 0; h < G; ++h, ++m) {
                if (!mbar_wait(&sm.bar[B_SFULL], m & 1, abort, 20)) { stop = true; break; }
                tc_fence_after();
                // this row's visible keys; a chunk fully visible to the warp's 32 rows needs no mask
                const int klo = max(i - L.W + 1, 0), khi = min(i, L.S - 1);
                auto chunk_full = [&](int kp0) {
                    return kp0 + 31 <= imin && kp0 > imax - L.W && kp0 >= 0 && kp0 + 31 < L.S;
                };
                float mu = sm.mref;
                if (!(mu <= 60.f)) {
                    float mx = -INFINITY;
#pragma unroll 1
                    for (int c8 = 0; c8 < 8; ++c8) {
                        const int kp0 = (c8 < 4 ? base0 : base1) + (c8 & 3) * 32;
                        const bool live = imin < L.S && kp0 <= imax && kp0 + 31 > imin - L.W && kp0 + 31 >= 0 && kp0 < L.S;
                        if (!live) continue;
                        float v[32];
                        tmem_ld32f(TM_S + lane_off + 32 * c8, v);
                        tmem_wait_ld();
                        if (chunk_full(kp0)) {
#pragma unroll
                            for (int e = 0; e < 32; ++e) mx = fmaxf(mx, v[e]);
                        } else {
                            const uint32_t vm = bit_range(klo - kp0, khi - kp0);
#pragma unroll
                            for (int e = 0; e < 32; ++e) mx = fmaxf(mx, ((vm >> e) & 1u) ? v[e] : -INFINITY);
                        }
                    }
                    mu = (mx == -INFINITY) ? 0.f : mx * c2;
                }
                float l = 0.f;
#pragma unroll 1
                for (int c8 = 0; c8 < 8; ++c8) {
                    const int kp0 = (c8 < 4 ? base0 : base1) + (c8 & 3) * 32;
                    const bool live = imin < L.S && kp0 <= imax && kp0 + 31 > imin - L.W && kp0 + 31 >= 0 && kp0 < L.S;
                    uint32_t pk[16];
                    if (live && chunk_full(kp0)) {
                        // every key visible to the warp's rows: no mask, scores two at a time
                        float v[32];
                        tmem_ld32f(TM_S + lane_off + 32 * c8, v);
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
                    } else if (live) {
                        float v[32];
                        tmem_ld32f(TM_S + lane_off + 32 * c8, v);
                        tmem_wait_ld();
                        const uint32_t vm = bit_range(klo - kp0, khi - kp0);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float p0 = fast_exp2(v[e] * c2 - mu), p1 = fast_exp2(v[e + 1] * c2 - mu);
                            p0 = ((vm >> e) & 1u) ? p0 : 0.f;  // (a masked score may overflow: selected away)
                            p1 = ((vm >> (e + 1)) & 1u) ? p1 : 0.f;
                            l += p0 + p1;
                            pk[e >> 1] = pack_bf16(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    }
                    tmem_st16(TM_P + lane_off + 16 * c8, pk);
                }
                tmem_wait_st();
                const int hg = st.kvh * G + h;
                if (i < L.S) p.lse[((size_t)st.b * L.Hq + hg) * L.S + i] = (mu + __log2f(l)) * kLn2;
                if (m >= 2 && !mbar_wait(&sm.bar[B_LEMPTY + (m & 1)], ((m >> 1) - 1) & 1, abort, 21)) { stop = true; break; }
                sm.rowinv[m & 1][r] = 1.f / l;
                mbar_arrive(&sm.bar[B_LFULL + (m & 1)]);
                tc_fence_before();
                mbar_arrive(&sm.bar[B_PFULL]);
            }
            if (stop) break;
        }
    } else if (warp >= 8 && warp < 12) {
        // ================================================ prologue: Q~ normalised + rotated in place
        // (K~ arrives converted from the preparation kernel)
        const int r = tid - 256;
        int m = 0;
        bool ok = true;
        for (int t = t_begin; t < t_end && ok; ++t) {
            const StepInfo st = decode_step(L, t, t_begin, t_end);
            if constexpr (!ANY) tf_angles(L, st.qb * TF_BM + r, sm.cs, r);  // this row's angles, shared by the G heads
            for (int h = 0; h < G; ++h, ++m) {
                const int buf = m & 1;
                if (!(ok = mbar_wait(&sm.bar[B_QFULL + buf], (m >> 1) & 1, abort, 33))) break;
                const float rinv =
                    ANY ? tf_prologue_row_any<true>(sm.Q[buf][0], sm.Q[buf][1], r, sm.gq, L, st.qb * TF_BM + r, oscale)
                        : tf_prologue_row<true>(sm.Q[buf][0], sm.Q[buf][1], r, sm.gq, L, sm.cs, oscale);
                fence_proxy_async_smem();
                if (p.save_q) {
                    // this warp's 32 rows of Q~ to the store the backward reads
                    const int hg = st.kvh * G + h, i = st.qb * TF_BM + r, wq = warp - 8;
                    const int row0 = st.qb * TF_BM + 32 * wq;
                    if (i < L.S) p.qrinv[((size_t)st.b * L.Hq + hg) * L.S + i] = rinv;
                    __syncwarp();
                    if (lane == 0 && row0 < L.S) {
                        tma_store_4d(&p.tm_q16s, sm.Q[buf][0] + wq * 32 * 128, 0, hg, row0, st.b);
                        tma_store_4d(&p.tm_q16s, sm.Q[buf][1] + wq * 32 * 128, 64, hg, row0, st.b);
                        tma_store_commit();
                    }
                }
                mbar_arrive(&sm.bar[B_QREADY + buf]);
                if (p.save_q && lane == 0) {
                    // the buffer is refilled (two heads on) only once the stores have read it
                    tma_store_wait_read();
                    mbar_arrive(&sm.bar[B_QSTORED + buf]);
                }
                __syncwarp();
            }
        }
    } else if (warp >= 12) {
        // ================================================ gate epilogue: out = sigmoid(g) * O / l
        // A warpgroup of its own, so the gate loads of head m are in flight while it waits
        // for head m's P.V to finish.
        const int r = tid - 384, wq = warp - 12;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        int e = 0;
        bool ok = true;
        for (int t = t_begin; t < t_end && ok; ++t) {
            const StepInfo st = decode_step(L, t, t_begin, t_end);
            const int i = st.qb * TF_BM + r;
            const bool valid = i < L.S;
            for (int h = 0; h < G; ++h, ++e) {
                const int buf = e & 1, hg = st.kvh * G + h;
                const size_t off = ((size_t)(st.b * (size_t)L.S + (valid ? i : 0)) * L.Hq + hg) * kD;
                uint4 gr[16];
                if (valid) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) gr[c] = __ldg(reinterpret_cast<const uint4*>(L.g + off) + c);
                }
                if (!(ok = mbar_wait(&sm.bar[B_OFULL + buf], (e >> 1) & 1, abort, 30))) break;
                if (!(ok = mbar_wait(&sm.bar[B_LFULL + buf], (e >> 1) & 1, abort, 31))) break;
                const float hi = 0.5f * sm.rowinv[buf][r];
                const float2 hinv = make_float2(hi, hi);
                mbar_arrive(&sm.bar[B_LEMPTY + buf]);
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld32(TM_O0 + buf * 128 + lane_off + 32 * c, v);
                    tmem_wait_ld();
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
                tc_fence_before();
                mbar_arrive(&sm.bar[B_OEMPTY + buf]);
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// 4-D 16-bit map {D, H, S, B} (innermost first), box {64, 1, rows, 1}, 128-byte swizzle
bool make_map(CUtensorMap* map, const void* base, int H, int S, int B,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, int rows = 128) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)S * H * kD * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

// Windows up to one key tile, any rotated dims and group size.  A shape test only: without
// the driver's tensor-map encoder the launch fails (ZGCM_ERR_CUDA).
bool fwd_tc_supported(const LayerParams& L) {
    return L.W <= TF_BN && L.S >= 1 && L.B >= 1;
}

size_t fwd_tc_smem_bytes() { return sizeof(FwdTcSmem) + 1024; }

cudaError_t launch_fwd_prep_k(const LayerParams& L, void* workspace, int* err_word, cudaStream_t stream,
                              float* krinv);

// fwd_prep_k_kernel (K~ into `workspace`, [B,S,Hkv,D] fp16), then the attention kernel.
// With `sv` (whose k16 the caller passes as `workspace`), both also keep the inverse RMS of
// every row, and the attention kernel stores Q~ for the backward.
cudaError_t launch_fwd_tc(const FwdParams& fp, void* workspace, int* err_word, cudaStream_t stream,
                          const SavedAct* sv) {
    FwdTcParams p;
    p.L = fp.L;
    p.out = fp.out;
    p.lse = fp.lse;
    p.err = err_word;
    p.save_q = sv ? 1 : 0;
    p.qrinv = sv ? sv->qrinv : nullptr;
    if (sv && !make_map(&p.tm_q16s, sv->q16, fp.L.Hq, fp.L.S, fp.L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 32))
        return cudaErrorInvalidValue;
    const int nqb = (fp.L.S + TF_BM - 1) / TF_BM;
    const long long total = (long long)fp.L.B * fp.L.Hkv * nqb;
    if (total > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.total_steps = (int)total;
    if (!make_map(&p.tm_q, fp.L.q, fp.L.Hq, fp.L.S, fp.L.B) ||
        !make_map(&p.tm_k16, workspace, fp.L.Hkv, fp.L.S, fp.L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_map(&p.tm_v, fp.L.v, fp.L.Hkv, fp.L.S, fp.L.B))
        return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = launch_fwd_prep_k(fp.L, workspace, err_word, stream, sv ? sv->krinv : nullptr);
    if (e != cudaSuccess) return e;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const size_t smem = fwd_tc_smem_bytes();
    auto kern = fp.L.rope_half == TF_HALF ? fwd_tc_kernel<false> : fwd_tc_kernel<true>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)(total < sms ? total : sms);
    kern<<<grid, TF_THREADS, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace zgcm
