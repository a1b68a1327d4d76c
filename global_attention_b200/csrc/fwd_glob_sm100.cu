// fwd_glob_sm100.cu — gated attention forward for windows wider than one key tile: the
// full-causal global layer (W >= S; ZGCM-1 layers 6/12/18/24/30) and any W > 128, on
// tcgen05 / TMEM / TMA (sm_100a).  Layer definition and page citations: common.cuh.
//
// Two kernels:
//   fwd_prep_k_kernel   K~ = fp16(RoPE(gamma_k * k / rms(k)) * oscale), one CTA per 128-row
//                       key tile, into the caller's workspace.  Same device function, angles
//                       and scale as the backward's preparation, so the scores below equal
//                       the backward's bit for bit.  (A key tile is read by every later query
//                       block; normalising it once here instead of in every CTA that reads it
//                       keeps the attention kernel's issue slots for the softmax.)
//   fwd_glob_tc_kernel  one CTA per unit (batch b, KV head, pair of query heads of its GQA
//                       group, 128-query block qb), heaviest blocks first.  The unit sweeps
//                       the key tiles kt_lo..qb of its window; K~ (fp16) and raw V (bf16)
//                       tiles stream through 2-slot TMA rings shared by both heads.
//
// TMEM (512 columns): S_a [0,128), S_b [128,256), O_a [256,384), O_b [384,512); P_x (bf16)
// is written over the front half of S_x.  Per key tile n and head x:
//   S_x(n) = Q~_x K~(n)^T     tcgen05.mma M=128 N=128 K=128, fp16 operands in smem
//   P_x(n) = exp2(S c2 - m_x) softmax warpgroup x (thread = query row), m_x a running
//                              reference raised only when a tile's max exceeds it by more
//                              than 2^8 (then O_x and l_x are rescaled in place)
//   O_x   += P_x(n) V(n)      tcgen05.mma M=128 N=128 K=128, P from TMEM, V MN-major
// The MMA warp issues PV_a(n), S_a(n+1), PV_b(n), S_b(n+1): while softmax a works on
// S_a(n+1) the tensor core runs head b's products and the other way round.  An MMA commit
// tracks every earlier MMA of the issuing thread, so S_x(n)'s completion also says that
// PV_x(n-1) is done and O_x may be rescaled.
// Epilogue (softmax warpgroups): out = sigmoid(g) * O / l, lse = (m + log2 l) ln 2.
//
// Warps (384 threads): w0 TMA producer, w1 MMA issuer + TMEM owner, w2-3 idle, w4-7
// softmax / epilogue of head a, w8-11 of head b.  Every wait is bounded; on expiry the CTA
// records the site, drains its copies and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include "tc_rows.cuh"

namespace zgcm {
using namespace sm100;

constexpr int FG_THREADS = 384;
constexpr int FG_SLOTS = 2;                 // K~ and V ring depth
constexpr float FG_RESCALE_LOG2 = 8.0f;     // P may reach 2^8 before the reference is raised

struct FwdGlobParams {
    CUtensorMap tm_q;    // raw q, bf16 {D, Hq, S, B}, box {64, 1, 128, 1}, 128B swizzle
    CUtensorMap tm_k;    // raw k, bf16 {D, Hkv, S, B} (preparation kernel)
    CUtensorMap tm_k16;  // K~ fp16 {D, Hkv, S, B} in the workspace
    CUtensorMap tm_v;    // raw v, bf16 {D, Hkv, S, B}
    LayerParams L;
    bf16* out;
    float* lse;
    int* err;
    float* krinv;        // inverse RMS of each k row, [B,Hkv,S] (preparation kernel; null = not kept)
    int units;           // B * Hkv * ceil(G / 2) * ceil(S / 128)
};

enum FgBar {
    FG_QFULL = 0, FG_QREADY = 2,
    FG_KFULL = 4, FG_KEMPTY = 4 + FG_SLOTS, FG_VFULL = 4 + 2 * FG_SLOTS, FG_VEMPTY = 4 + 3 * FG_SLOTS,
    FG_SFULL = 4 + 4 * FG_SLOTS, FG_PFULL = FG_SFULL + 2, FG_OFULL = FG_PFULL + 2,
    FG_DONE = FG_OFULL + 2, FG_COUNT = FG_DONE + 1
};

struct FwdGlobSmem {
    alignas(1024) unsigned char Q[2][2][TF_HALF_BYTES];          // [head][d-half]: raw q -> Q~ fp16
    alignas(1024) unsigned char K[FG_SLOTS][2][TF_HALF_BYTES];   // [slot][d-half]: K~ fp16
    alignas(1024) unsigned char V[FG_SLOTS][2][TF_HALF_BYTES];   // [slot][d-half]: raw v bf16
    float gq[kD], gk[kD];
    uint64_t bar[FG_COUNT];
    uint32_t tmem_base;
    int abort;
};

struct FgUnit {
    int b, kvh, h0, h1, qb, kt_lo, n_tiles;   // h0, h1: the unit's two query heads
};

// Unit u, heaviest first: the query block runs from the last one down (to the block of the
// first query row, q_off / 128); the head pairs of a KV group are adjacent so that the CTAs
// reading the same K/V tiles run together.  With an odd
// number of heads per KV head the last pair repeats the last head (its two warpgroups compute,
// and write, the same rows).
__device__ __forceinline__ FgUnit fg_unit(const LayerParams& L, int u) {
    const int nqb = (L.S + TF_BM - 1) / TF_BM;
    const int npair = (L.G + 1) / 2, per_qb = L.B * L.Hkv * npair;
    FgUnit w;
    w.qb = nqb - 1 - u / per_qb;
    const int rest = u - (nqb - 1 - w.qb) * per_qb;
    const int hp = rest % npair;
    w.kvh = (rest / npair) % L.Hkv;
    w.b = rest / (npair * L.Hkv);
    w.h0 = w.kvh * L.G + 2 * hp;
    w.h1 = w.kvh * L.G + min(2 * hp + 1, L.G - 1);
    const int q0 = w.qb * TF_BM;
    // first key tile holding a key visible to the block's first row: j > q0 - W
    w.kt_lo = (L.W >= L.S || q0 - L.W + 1 <= 0) ? 0 : (q0 - L.W + 1) / TF_BN;
    w.n_tiles = w.qb - w.kt_lo + 1;
    return w;
}

// ------------------------------------------------------------------ K~ preparation

constexpr int FP_THREADS = 128;

struct FwdPrepSmem {
    alignas(1024) unsigned char X[2][TF_HALF_BYTES];
    float gq[kD], gk[kD];
    uint64_t bar;
};

// One CTA per 128-row key tile (b, KV head, t): raw k -> K~ fp16 in place -> workspace.
// ANY: any number of rotated pairs, the angles formed as needed (else the layer's 21, in registers)
template <bool ANY>
__global__ void __launch_bounds__(FP_THREADS, 4) fwd_prep_k_kernel(const __grid_constant__ FwdGlobParams p) {
    const LayerParams& L = p.L;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    FwdPrepSmem& sm = *reinterpret_cast<FwdPrepSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int r = threadIdx.x;
    const int nt = (L.S + TF_BN - 1) / TF_BN;
    const int t = (int)blockIdx.x % nt, chain = (int)blockIdx.x / nt;
    const int h = chain % L.Hkv, b = chain / L.Hkv;
    volatile int abort = 0;
    if (r == 0) {
        mbar_init(&sm.bar, 1);
        fence_barrier_init();
    }
    sm.gq[r] = L.gamma_q[r];
    sm.gk[r] = L.gamma_k[r];
    __syncthreads();
    if (r == 0) {
        mbar_expect_tx(&sm.bar, TF_TILE_BYTES);
        tma_load_4d(sm.X[0], &p.tm_k, &sm.bar, 0, h, t * TF_BN, b);
        tma_load_4d(sm.X[1], &p.tm_k, &sm.bar, 64, h, t * TF_BN, b);
    }
    const int pos = t * TF_BN + r;
    float2 csr[ANY ? 1 : TF_HALF];
    if constexpr (!ANY) {
#pragma unroll
        for (int q = 0; q < TF_HALF; ++q) rope_cs(L.theta[q], pos, csr[q].x, csr[q].y);
    }
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    const bool ok = __syncthreads_and(mbar_wait(&sm.bar, 0, &abort, 260)) != 0;
    if (ok) {
        float rinv;
        if constexpr (ANY)
            rinv = tf_prologue_row_any<true>(sm.X[0], sm.X[1], r, sm.gk, L, pos, oscale);
        else
            rinv = tf_prologue_row_at<true>(sm.X[0], sm.X[1], r, sm.gk, L, [&](int q) { return csr[q]; }, oscale);
        if (p.krinv && pos < L.S) p.krinv[(size_t)chain * L.S + pos] = rinv;
        fence_proxy_async_smem();
    } else if (r == 0) {
        mbar_wait_drain(&sm.bar, 0);
    }
    __syncthreads();
    if (r == 0) {
        if (ok) {
            tma_store_4d(&p.tm_k16, sm.X[0], 0, h, t * TF_BN, b);
            tma_store_4d(&p.tm_k16, sm.X[1], 64, h, t * TF_BN, b);
            tma_store_commit();
            tma_store_wait_read();
        } else if (p.err) {
            atomicExch(p.err, 260);
        }
    }
}

// ------------------------------------------------------------------ attention kernel

template <bool ANY>
__global__ void __launch_bounds__(FG_THREADS, 1) fwd_glob_tc_kernel(const __grid_constant__ FwdGlobParams p) {
    const LayerParams& L = p.L;
    extern __shared__ unsigned char smem_raw[];
    FwdGlobSmem& sm = *reinterpret_cast<FwdGlobSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &sm.abort;
    const FgUnit w = fg_unit(L, (int)blockIdx.x);
    const int q0 = w.qb * TF_BM;

    if (tid == 0) {
        sm.abort = 0;
        for (int x = 0; x < 2; ++x) {
            mbar_init(&sm.bar[FG_QFULL + x], 1);
            mbar_init(&sm.bar[FG_QREADY + x], 128);
            mbar_init(&sm.bar[FG_SFULL + x], 1);
            mbar_init(&sm.bar[FG_PFULL + x], 128);
            mbar_init(&sm.bar[FG_OFULL + x], 1);
        }
        for (int s = 0; s < FG_SLOTS; ++s) {
            mbar_init(&sm.bar[FG_KFULL + s], 1);
            mbar_init(&sm.bar[FG_KEMPTY + s], 1);
            mbar_init(&sm.bar[FG_VFULL + s], 1);
            mbar_init(&sm.bar[FG_VEMPTY + s], 1);
        }
        mbar_init(&sm.bar[FG_DONE], 1);
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
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k16);
        prefetch_tmap(&p.tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    const float c2 = L.scale_log2 / (oscale * oscale);  // S holds oscale^2 q~.k~

    // register budgets (set inside each role's branch): warpgroup 0 56, softmax warpgroups 224;
    // 128 * 56 + 256 * 224 = 384 * 168, the launch's allocation
    if (warp == 0) {
        // ================================================ TMA producer: Q tiles, then the K~ / V ring
        reg_dealloc<56>();
        if (lane == 0) {
            for (int x = 0; x < 2; ++x) {
                mbar_expect_tx(&sm.bar[FG_QFULL + x], TF_TILE_BYTES);
                // (q holds the rows from position q_off on)
                tma_load_4d(sm.Q[x][0], &p.tm_q, &sm.bar[FG_QFULL + x], 0, x ? w.h1 : w.h0, q0 - L.q_off, w.b);
                tma_load_4d(sm.Q[x][1], &p.tm_q, &sm.bar[FG_QFULL + x], 64, x ? w.h1 : w.h0, q0 - L.q_off, w.b);
            }
            int nk = 0, nv = 0;  // K~ / V tiles issued
            for (int n = 0; n < w.n_tiles; ++n) {
                const int s = n % FG_SLOTS, ph = (n / FG_SLOTS) & 1, k0 = (w.kt_lo + n) * TF_BN;
                if (n >= FG_SLOTS && !mbar_wait(&sm.bar[FG_KEMPTY + s], ph ^ 1, abort, 270)) break;
                mbar_expect_tx(&sm.bar[FG_KFULL + s], TF_TILE_BYTES);
                tma_load_4d(sm.K[s][0], &p.tm_k16, &sm.bar[FG_KFULL + s], 0, w.kvh, k0, w.b);
                tma_load_4d(sm.K[s][1], &p.tm_k16, &sm.bar[FG_KFULL + s], 64, w.kvh, k0, w.b);
                nk = n + 1;
                if (n >= FG_SLOTS && !mbar_wait(&sm.bar[FG_VEMPTY + s], ph ^ 1, abort, 271)) break;
                mbar_expect_tx(&sm.bar[FG_VFULL + s], TF_TILE_BYTES);
                tma_load_4d(sm.V[s][0], &p.tm_v, &sm.bar[FG_VFULL + s], 0, w.kvh, k0, w.b);
                tma_load_4d(sm.V[s][1], &p.tm_v, &sm.bar[FG_VFULL + s], 64, w.kvh, k0, w.b);
                nv = n + 1;
            }
            // every copy issued must land before the CTA exits (matters after an abort)
            for (int x = 0; x < 2; ++x) mbar_wait_drain(&sm.bar[FG_QFULL + x], 0);
            for (int n = nk > FG_SLOTS ? nk - FG_SLOTS : 0; n < nk; ++n)
                mbar_wait_drain(&sm.bar[FG_KFULL + n % FG_SLOTS], (n / FG_SLOTS) & 1);
            for (int n = nv > FG_SLOTS ? nv - FG_SLOTS : 0; n < nv; ++n)
                mbar_wait_drain(&sm.bar[FG_VFULL + n % FG_SLOTS], (n / FG_SLOTS) & 1);
        }
    } else if (warp == 1) {
        // ================================================ MMA issuer
        reg_dealloc<56>();
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_f16(128, 128, false);
            constexpr uint32_t IDESC_O = idesc_bf16(128, 128, true);
            const uint32_t q_base = smem_u32(sm.Q[0][0]);
            const uint32_t k_base = smem_u32(sm.K[0][0]);
            const uint32_t v_base = smem_u32(sm.V[0][0]);
            auto issue_s = [&](int x, int n) {
                const int s = n % FG_SLOTS;
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * TF_HALF_BYTES + (kk & 3) * 32;
                    const uint64_t a = sdesc_sw128(q_base + x * 2 * TF_HALF_BYTES + off, 16, 1024);
                    const uint64_t bd = sdesc_sw128(k_base + s * 2 * TF_HALF_BYTES + off, 16, 1024);
                    mma_ss(tmem + 128 * x, a, bd, IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar[FG_SFULL + x]);
            };
            auto issue_pv = [&](int x, int n) {
                const int s = n % FG_SLOTS;
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bd = sdesc_sw128(v_base + s * 2 * TF_HALF_BYTES + kk * 16 * 128, TF_HALF_BYTES, 1024);
                    mma_ts(tmem + 256 + 128 * x, tmem + 128 * x + kk * 8, bd, IDESC_O, (n > 0 || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(&sm.bar[FG_QREADY + 0], 0, abort, 280) &&
                      mbar_wait(&sm.bar[FG_QREADY + 1], 0, abort, 281) &&
                      mbar_wait(&sm.bar[FG_KFULL + 0], 0, abort, 282);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
                mma_commit(&sm.bar[FG_KEMPTY + 0]);
            }
            for (int n = 0; n < w.n_tiles && ok; ++n) {
                const int s = n % FG_SLOTS, ph = (n / FG_SLOTS) & 1;
                const bool more = n + 1 < w.n_tiles;
                const int s1 = (n + 1) % FG_SLOTS, ph1 = ((n + 1) / FG_SLOTS) & 1;
                if (!(ok = mbar_wait(&sm.bar[FG_VFULL + s], ph, abort, 283))) break;
                for (int x = 0; x < 2 && ok; ++x) {
                    if (!(ok = mbar_wait(&sm.bar[FG_PFULL + x], n & 1, abort, 285 + x))) break;
                    tc_fence_after();
                    issue_pv(x, n);
                    if (!more) {
                        mma_commit(&sm.bar[FG_OFULL + x]);
                        continue;
                    }
                    if (x == 0 && !(ok = mbar_wait(&sm.bar[FG_KFULL + s1], ph1, abort, 284))) break;
                    issue_s(x, n + 1);
                }
                if (!ok) break;
                mma_commit(&sm.bar[FG_VEMPTY + s]);
                if (more) mma_commit(&sm.bar[FG_KEMPTY + s1]);
            }
            // every MMA issued must complete before TMEM is released
            mma_commit(&sm.bar[FG_DONE]);
            if (!mbar_wait(&sm.bar[FG_DONE], 0, abort, 287)) mbar_wait_drain(&sm.bar[FG_DONE], 0);
        }
    } else if (warp < 4) {
        reg_dealloc<56>();  // warps 2-3: idle
    } else {
        // ================================================ softmax + epilogue of head x (thread = query row)
        reg_alloc<224>();
        const int x = (warp - 4) >> 2, wq = warp & 3;
        const int r = 32 * wq + lane, i = q0 + r, hx = x ? w.h1 : w.h0;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        const uint32_t TM_S = tmem + 128 * x, TM_O = tmem + 256 + 128 * x;
        bool ok = mbar_wait(&sm.bar[FG_QFULL + x], 0, abort, 290);
        if (ok) {
            // Q~_x in place: the same device function, angles and scale as the backward's Q~
            if constexpr (ANY) {
                tf_prologue_row_any<true>(sm.Q[x][0], sm.Q[x][1], r, sm.gq, L, i, oscale);
            } else {
                float2 csr[TF_HALF];
#pragma unroll
                for (int t = 0; t < TF_HALF; ++t) rope_cs(L.theta[t], i, csr[t].x, csr[t].y);
                tf_prologue_row_at<true>(sm.Q[x][0], sm.Q[x][1], r, sm.gq, L, [&](int t) { return csr[t]; }, oscale);
            }
            fence_proxy_async_smem();
            mbar_arrive(&sm.bar[FG_QREADY + x]);
        }
        // visible keys of row i: lo <= j <= hi
        const int lo = max(i - L.W + 1, 0), hi = i;
        const int rmin = q0 + 32 * wq, rmax = rmin + 31;  // rows of this warp
        float m_ref = -INFINITY, l = 0.f;
        for (int n = 0; n < w.n_tiles && ok; ++n) {
            const int k0 = (w.kt_lo + n) * TF_BN;
            if (!(ok = mbar_wait(&sm.bar[FG_SFULL + x], n & 1, abort, 291))) break;
            tc_fence_after();
            float v[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32f(TM_S + lane_off + 32 * c, v + 32 * c);
            tmem_wait_ld();
            // a tile is fully visible to the warp's rows unless it crosses the diagonal or the
            // window's lower edge (warp-uniform test)
            const bool full = k0 + TF_BN - 1 <= rmin && k0 > rmax - L.W;
            if (!full) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t vm = bit_range(lo - (k0 + 32 * c), hi - (k0 + 32 * c));
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[32 * c + e] = ((vm >> e) & 1u) ? v[32 * c + e] : -INFINITY;
                }
            }
            // row max and (below) row sum over 8 and 4 independent partials: a single running
            // value would make each a chain of dependent instructions as long as the row
            float mx8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mx8[k] = v[k];
#pragma unroll
            for (int e = 8; e < 128; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], v[e]);
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            const float mt = mx * c2;   // -inf when the row sees no key of this tile
            const bool raise = mt > m_ref + FG_RESCALE_LOG2;
            const bool warp_raise = __any_sync(0xffffffffu, raise) != 0;
            // alpha = 2^(m_old - m_new) for a raised row (0 from an empty start), 1 otherwise
            const float alpha = raise ? fast_exp2(m_ref - mt) : 1.0f;
            if (raise) m_ref = mt;
            l *= alpha;
            const float mb = m_ref == -INFINITY ? 0.f : m_ref;
            // scores two at a time (paired fp32 instructions), the sum in two paired partials
            const float2 cc = make_float2(c2, c2), nb = make_float2(-mb, -mb);
            float2 la = make_float2(0.f, 0.f), lb = la;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float2 xa = ffma2(make_float2(v[32 * c + e], v[32 * c + e + 1]), cc, nb);
                    const float2 xb = ffma2(make_float2(v[32 * c + e + 2], v[32 * c + e + 3]), cc, nb);
                    const float2 pa = make_float2(fast_exp2(xa.x), fast_exp2(xa.y));
                    const float2 pb = make_float2(fast_exp2(xb.x), fast_exp2(xb.y));
                    la = fadd2(la, pa);
                    lb = fadd2(lb, pb);
                    pk[e >> 1] = pack_bf16(pa.x, pa.y);
                    pk[(e >> 1) + 1] = pack_bf16(pb.x, pb.y);
                }
                tmem_st16(TM_S + lane_off + 16 * c, pk);
            }
            l += (la.x + la.y) + (lb.x + lb.y);
            if (warp_raise && n > 0) {
                // O_x holds PV_x(0..n-1), complete (S_x(n) was issued after PV_x(n-1))
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float o[32];
                    tmem_ld32f(TM_O + lane_off + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= alpha;
                    tmem_st32f(TM_O + lane_off + 32 * c, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar[FG_PFULL + x]);
        }
        // ------------------------------------------ epilogue: out = sigmoid(g) * O / l, lse
        const bool valid = i < L.S;
        const int iq = valid ? i - L.q_off : 0;  // row of the query-side tensors
        const size_t off = ((size_t)(w.b * (size_t)L.Sq + iq) * L.Hq + hx) * kD;
        uint4 gr[16];
        if (valid) {
#pragma unroll
            for (int c = 0; c < 16; ++c) gr[c] = __ldg(reinterpret_cast<const uint4*>(L.g + off) + c);
        }
        if (ok && (ok = mbar_wait(&sm.bar[FG_OFULL + x], 0, abort, 292))) {
            tc_fence_after();
            const float inv = 1.0f / l;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(TM_O + lane_off + 32 * c, o);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const uint4 g4 = gr[4 * c + q4];
                        const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
                        uint32_t ow[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const float2 gf = unpack_bf16(gw[e2]);
                            // sigmoid(x) = 0.5 + 0.5 tanh(x / 2)
                            const float s0 = fmaf(0.5f, fast_tanh(0.5f * gf.x), 0.5f);
                            const float s1 = fmaf(0.5f, fast_tanh(0.5f * gf.y), 0.5f);
                            const int col = 8 * q4 + 2 * e2;
                            ow[e2] = pack_bf16(s0 * (__uint_as_float(o[col]) * inv),
                                               s1 * (__uint_as_float(o[col + 1]) * inv));
                        }
                        *reinterpret_cast<uint4*>(p.out + off + 32 * c + 8 * q4) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
            }
            if (valid) p.lse[((size_t)w.b * L.Hq + hx) * L.Sq + iq] = (m_ref + __log2f(l)) * kLn2;
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode_g() {
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

// 4-D 16-bit map {D, H, S, B} (innermost first), box {64, 1, 128, 1}, 128-byte swizzle
bool make_map_g(CUtensorMap* map, const void* base, int H, int S, int B, CUtensorMapDataType dtype) {
    auto enc = get_encode_g();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)S * H * kD * 2};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Windows wider than one key tile (W > 128, including the global layer W >= S): any number of
// rotated dims and of query heads per KV head.  A shape test only: without the driver's
// tensor-map encoder the launch fails (ZGCM_ERR_CUDA).
bool fwd_glob_supported(const LayerParams& L) {
    return L.W > TF_BN && L.S >= 1 && L.B >= 1;
}

// K~ fp16 [B, S, Hkv, D] (both tcgen05 forwards)
size_t fwd_glob_workspace_bytes(int B, int S, int Hkv) { return (size_t)B * S * Hkv * kD * 2; }

cudaError_t launch_prep_q_only(const LayerParams& L, void* q16, float* qrinv, int* err_word, cudaStream_t stream);

// With `sv`, K~ goes to sv->k16 (the caller passes it as `workspace`) with each k row's
// inverse RMS, and a preparation pass leaves Q~ and the q rows' inverse RMS there too.
cudaError_t launch_fwd_glob_tc(const FwdParams& fp, void* workspace, int* err_word, cudaStream_t stream,
                               const SavedAct* sv) {
    FwdGlobParams p;
    p.L = fp.L;
    p.krinv = sv ? sv->krinv : nullptr;
    // a window of S or more is the full causal one: clamped so that window arithmetic stays in range
    if (p.L.W > p.L.S) p.L.W = p.L.S;
    const LayerParams& L = p.L;
    p.out = fp.out;
    p.lse = fp.lse;
    p.err = err_word;
    const long long nqb = (L.S + TF_BM - 1) / TF_BM;
    // query blocks from the one of the first query row (q_off, a multiple of 128) on
    const long long units = (long long)L.B * L.Hkv * ((L.G + 1) / 2) * (nqb - L.q_off / TF_BM);
    const long long k_tiles = (long long)L.B * L.Hkv * nqb;
    if (units > 0x7fffffffLL || k_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.units = (int)units;
    if (!make_map_g(&p.tm_q, L.q, L.Hq, L.Sq, L.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
        !make_map_g(&p.tm_k, L.k, L.Hkv, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
        !make_map_g(&p.tm_k16, workspace, L.Hkv, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_map_g(&p.tm_v, L.v, L.Hkv, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
        return cudaErrorInvalidValue;
    const size_t smem_p = sizeof(FwdPrepSmem) + 1024, smem_a = sizeof(FwdGlobSmem) + 1024;
    const bool any = L.rope_half != TF_HALF;
    auto prep = any ? fwd_prep_k_kernel<true> : fwd_prep_k_kernel<false>;
    auto attn = any ? fwd_glob_tc_kernel<true> : fwd_glob_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_p);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a);
    if (e != cudaSuccess) return e;
    prep<<<(int)k_tiles, FP_THREADS, smem_p, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (sv && (e = launch_prep_q_only(fp.L, sv->q16, sv->qrinv, err_word, stream)) != cudaSuccess) return e;
    attn<<<(int)units, FG_THREADS, smem_a, stream>>>(p);
    return cudaGetLastError();
}

// K~ fp16 of every key tile into `workspace` ([B,S,Hkv,D]) for the sliding-window forward.
// With `krinv`, also each k row's inverse RMS ([B,Hkv,S]).
cudaError_t launch_fwd_prep_k(const LayerParams& L, void* workspace, int* err_word, cudaStream_t stream,
                              float* krinv) {
    FwdGlobParams p;
    p.L = L;
    p.krinv = krinv;
    p.out = nullptr;
    p.lse = nullptr;
    p.err = err_word;
    p.units = 0;
    const long long k_tiles = (long long)L.B * L.Hkv * ((L.S + TF_BN - 1) / TF_BN);
    if (k_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (!make_map_g(&p.tm_k, L.k, L.Hkv, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
        !make_map_g(&p.tm_k16, workspace, L.Hkv, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return cudaErrorInvalidValue;
    const size_t smem_p = sizeof(FwdPrepSmem) + 1024;
    auto prep = L.rope_half != TF_HALF ? fwd_prep_k_kernel<true> : fwd_prep_k_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_p);
    if (e != cudaSuccess) return e;
    prep<<<(int)k_tiles, FP_THREADS, smem_p, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace zgcm
