// bwd_sm100.cu — gated sliding-window attention backward on tcgen05 / TMEM / TMA (sm_100a).
//
// Exact gradients of L = sum(dout * out) for the ZGCM-1 layer (definition and page
// citations in common.cuh), for windows W <= 128 (wider ones: bwd_glob_sm100.cu with the
// key-major kernel here in its wide mode).  Every kernel that rotates comes in two instances:
// the layer's 21 rotated pairs, unrolled, and any other number (the angles formed where
// needed).  The gate pass, the preparation passes (bwd_prep_kv,
// bwd_prep_q: fp16 K~, V, Q~ with the rows' inverse RMS; bwd_prep_v alone when the forward
// kept Q~ and K~) and the two score kernels:
//
//   bwd_gate   streaming pass over dout, g, out (coalesced, 16 lanes per row): the gate
//              backward dg = dout*out*(1-sigmoid(g)), and dA = dout*sigmoid(g) stored as fp16
//              scaled by a power of two per row (2^-e and max|dout| saved per row).
//   bwd_q_tc   query-major sweep over (b, KV head, 128-query block) steps, all query heads
//              of the group per step, key tiles qb-1 and qb in a 2-slot ring (as the forward).
//              Per head: S = Q~ K~^T and dP = dA V^T (both M=128 N=256 into TMEM, issued
//              step by step in turn), then one
//              warpgroup per row forms the log-sum-exp, Delta = sum_j P dP and dS = P(dP-Delta)
//              from its own scores, dQ~ = dS K~ (M=128 N=128 K=256, dS from TMEM), and an
//              epilogue warpgroup applies the RoPE / RMSNorm backward and writes dq.  Writes
//              lse and Delta per row.
//   bwd_kv_tc  key-major: persistent CTAs over (b, KV head, 128-key tile) units; per unit the
//              Hq/Hkv heads x the two query blocks that see the tile:
//              S^T = K~ Q~^T, dP^T = V dA^T, P^T and dS^T from the saved lse and Delta,
//              dV += P^T dA and dK~ += dS^T Q~ accumulated in TMEM; epilogue writes dv and dk
//              (RoPE / RMSNorm backward).
//
// Numerics.  Every product runs as kind::f16 with fp16 operands (11-bit significand) and
// fp32 accumulation; each operand is brought into fp16 range by an exact power-of-two scale
// that the product lets factor out: q~, k~ are RMS-normalised (one scale from gamma); dA
// rows (undone per row in dP, per column in dP^T); dS rows of the query-major products; V and
// dS^T rows of the key-major products; in dV = P^T dA the dA row scales are moved onto the
// columns of P^T relative to one scale per unit (a sum over query rows).  Scales are undone
// in fp32.  Measured in a CPU emulation against the fp64 oracle this keeps every gradient
// within the bf16 output rounding of the reference (single bf16 operands did not).
#include "bwd_tc.cuh"

namespace zgcm {

// =====================================================================  gate backward pass

constexpr int GATE_THREADS = 256;
constexpr int GATE_UNROLL = 2;  // rows in flight per half-warp

// Sigmoid gate backward of out = sigmoid(g) * A (the gated-attention page, output gate):
//   dA = dout * sigmoid(g)  -> da16 = fp16(dA * 2^e), e = fit_exp(max|dout| of the row)
//   dg = dout * A * sigmoid'(g) = dout * out * (1 - sigmoid(g))
// One half-warp per row of D = 128 (16 lanes x 8 values, fully coalesced), GATE_UNROLL rows
// per half-warp in flight; every loop bound is warp-uniform so the row-max shuffles see all
// 32 lanes.  dainv = 2^-e (0 when the row of dout is all zero: its dA row is zero and must
// not be rescaled), domax = max|dout|, both [B,Hq,Spad] (row_stride; the query-major kernel
// fills the entries past S).  With DELTA (wide windows) also Delta = sum_d dout*out
// per row, [B,Hq,Spad]: the row sum of dA * A (A = out / sigmoid(g)), which the wide-window
// query-major kernel needs before its first key tile.
// Rows: dout, g, out, dg are [B,Sq,Hq,D] (positions q_off .. S-1, Sq = S - q_off); da16 and
// the row arrays are indexed by position ([B,S,Hq,D], [B,Hq,Spad]).
template <bool DELTA>
__global__ void __launch_bounds__(GATE_THREADS, 4) bwd_gate_kernel(const bf16* __restrict__ dout,
                                                                const bf16* __restrict__ g,
                                                                const bf16* __restrict__ out,
                                                                bf16* __restrict__ dg, __half* __restrict__ da16,
                                                                float* __restrict__ dainv,
                                                                float* __restrict__ domax,
                                                                float* __restrict__ delta, long long rows, int S,
                                                                int Hq, int q_off) {
    const int Sq = S - q_off;
    const int lane = threadIdx.x & 31, sub = lane & 15;
    const long long warp0 = ((long long)blockIdx.x * GATE_THREADS + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * GATE_THREADS) >> 5;
    const long long stride = 2 * nwarps;  // rows between the k-th rows of consecutive unroll slots
    for (long long base = 2 * warp0; base < rows; base += GATE_UNROLL * stride) {
        uint4 ud[GATE_UNROLL], ug[GATE_UNROLL], uo[GATE_UNROLL];
#pragma unroll
        for (int k = 0; k < GATE_UNROLL; ++k) {
            const long long r = base + k * stride + (lane >> 4);
            ud[k] = ug[k] = uo[k] = make_uint4(0u, 0u, 0u, 0u);
            if (r < rows) {
                const size_t o = (size_t)r * (kD / 8) + sub;
                ud[k] = __ldg(reinterpret_cast<const uint4*>(dout) + o);
                ug[k] = __ldg(reinterpret_cast<const uint4*>(g) + o);
                uo[k] = __ldg(reinterpret_cast<const uint4*>(out) + o);
            }
        }
#pragma unroll
        for (int k = 0; k < GATE_UNROLL; ++k) {
            const long long r = base + k * stride + (lane >> 4);
            const uint32_t wd[4] = {ud[k].x, ud[k].y, ud[k].z, ud[k].w};
            const uint32_t wg[4] = {ug[k].x, ug[k].y, ug[k].z, ug[k].w};
            const uint32_t wo[4] = {uo[k].x, uo[k].y, uo[k].z, uo[k].w};
            float mx = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fd = unpack_bf16(wd[e]);
                mx = fmaxf(mx, fmaxf(fabsf(fd.x), fabsf(fd.y)));
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const int ea = fit_exp(mx);
            const float sc = ldexpf(1.0f, ea);
            uint32_t da[4], dgw[4];
            float dsum = 0.f;  // sum_d dout out = sum_d dA A  (Delta of the wide-window backward)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fd = unpack_bf16(wd[e]), fg = unpack_bf16(wg[e]), fo = unpack_bf16(wo[e]);
                const float s0 = sigmoidf_(fg.x), s1 = sigmoidf_(fg.y);
                da[e] = pack2<true>(fd.x * s0 * sc, fd.y * s1 * sc);
                dgw[e] = pack_bf16(fd.x * fo.x * (1.f - s0), fd.y * fo.y * (1.f - s1));
                if constexpr (DELTA) dsum = fmaf(fd.x, fo.x, fmaf(fd.y, fo.y, dsum));
            }
            if constexpr (DELTA) {
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
            }
            if (r < rows) {
                // row r = (b*Sq + s)*Hq + h is position s + q_off: [B,Hq,Spad] index
                // (b*Hq + h)*Spad + s + q_off, da16 row (b*S + s + q_off)*Hq + h (32-bit
                // division where the row count allows: the 64-bit one is a long sequence)
                size_t ro = 0, rda = (size_t)r;
                if (q_off || sub == 0) {
                    if (rows <= 0xffffffffLL) {
                        const uint32_t ru = (uint32_t)r, sh = (uint32_t)Sq * (uint32_t)Hq;
                        const uint32_t b = ru / sh, rem = ru - b * sh;
                        const uint32_t s = rem / (uint32_t)Hq, h = rem - s * (uint32_t)Hq;
                        ro = ((size_t)b * Hq + h) * row_stride(S) + s + q_off;
                        if (q_off) rda = ((size_t)b * S + s + q_off) * Hq + h;
                    } else {
                        const long long sh = (long long)Sq * Hq;
                        const long long b = r / sh, rem = r - b * sh;
                        const long long s = rem / Hq, h = rem - s * Hq;
                        ro = (size_t)(b * Hq + h) * row_stride(S) + s + q_off;
                        if (q_off) rda = ((size_t)b * S + s + q_off) * Hq + h;
                    }
                }
                reinterpret_cast<uint4*>(da16)[rda * (kD / 8) + sub] = make_uint4(da[0], da[1], da[2], da[3]);
                reinterpret_cast<uint4*>(dg)[(size_t)r * (kD / 8) + sub] = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
                if (sub == 0) {
                    dainv[ro] = mx > 0.f ? 1.0f / sc : 0.f;
                    domax[ro] = mx;
                    if constexpr (DELTA) delta[ro] = dsum;
                }
            }
        }
    }
}

// Query-major pass over one 32-key chunk of a row (S, dP as accumulated in TMEM), with
// vm = the visible keys of the chunk (ignored when FULL: all visible):
//   P = 2^(s c2 - lse2) on visible keys (0 elsewhere) and P dv, dv = dP before the chunk's
//   scale kd (the caller applies kd to the chunk sums): cnum += P dv, cmpd = max |P dv|,
//   csa += P dv s, sb += P s.  P and P dv replace s and dv in place (written back to TMEM).
template <bool FULL>
__device__ __forceinline__ void q_pass1_chunk(float (&sv)[32], float (&dv)[32], uint32_t vm, float c2, float lse2,
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

// Key-major chunk: one key row j against 32 query columns i0.. (S^T, dP^T from TMEM; per
// column lse (base 2), Delta and dA row scale 2^-e_i from shared memory; vm = the visible
// columns, ignored when FULL):
//   P^T = 2^(s c2 - lse) (visible pairs), dP^T = dv * vin * 2^-e_i,
//   P^T for dV carries 2^(E - e_i) (su = 2^E), dS^T = P^T (dP^T - Delta) * dsc,
//   kacc += dS^T S^T (unscaled dS^T; dk's RMSNorm row term).
template <bool FULL>
__device__ __forceinline__ void kv_chunk(const float* sv, const float* dv, const float* lse2c, const float* deltac,
                                         const float* dcolc, uint32_t vm, float vin, float su, float dsc, float c2,
                                         uint32_t (&pp)[16], uint32_t (&dd)[16], float& kacc) {
    // two query columns per paired fp32 instruction
    const float2 cc = make_float2(c2, c2), vin2 = make_float2(vin, vin), su2 = make_float2(su, su),
                 dsc2 = make_float2(dsc, dsc);
    float2 kacc2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int e4 = 0; e4 < 8; ++e4) {
        const float4 ls = *reinterpret_cast<const float4*>(lse2c + 4 * e4);
        const float4 dl = *reinterpret_cast<const float4*>(deltac + 4 * e4);
        const float4 dc = *reinterpret_cast<const float4*>(dcolc + 4 * e4);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int e = 4 * e4 + 2 * hf;
            const float2 lsp = hf ? make_float2(ls.z, ls.w) : make_float2(ls.x, ls.y);
            const float2 dlp = hf ? make_float2(dl.z, dl.w) : make_float2(dl.x, dl.y);
            const float2 dcp = hf ? make_float2(dc.z, dc.w) : make_float2(dc.x, dc.y);
            const float2 s = make_float2(sv[e], sv[e + 1]);
            const float2 x = fsub2(fmul2(s, cc), lsp);
            float2 pv = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            if (!FULL) {  // (columns past the sequence: masked)
                pv.x = ((vm >> e) & 1u) ? pv.x : 0.f;
                pv.y = ((vm >> (e + 1)) & 1u) ? pv.y : 0.f;
            }
            const float2 dp = fmul2(fmul2(make_float2(dv[e], dv[e + 1]), vin2), dcp);
            const float2 d = fmul2(pv, fsub2(dp, dlp));
            kacc2 = ffma2(d, s, kacc2);
            const float2 p2 = fmul2(pv, fmul2(dcp, su2));
            const float2 d2 = fmul2(d, dsc2);
            pp[2 * e4 + hf] = pack2<true>(p2.x, p2.y);
            dd[2 * e4 + hf] = pack2<true>(d2.x, d2.y);
        }
    }
    kacc += kacc2.x + kacc2.y;
}

// =====================================================================  query-major kernel

enum QBar {
    QB_KFULL = 0, QB_KEMPTY = 4, QB_VFULL = 6, QB_VEMPTY = 10,
    QB_QFULL = 12, QB_QEMPTY = 14, QB_DAEMPTY = 15,
    QB_DSFULL = 17, QB_DQFULL = 18, QB_DQEMPTY = 19, QB_DONE = 20, QB_DAFULL = 21,
    QB_DPFULL = 22, QB_COUNT = 23
};

struct BwdQTcSmem {
    alignas(1024) unsigned char K[2][TF_RING_HALF];    // K~ fp16, 2-slot ring split by d-half
    alignas(1024) unsigned char V[2][TF_RING_HALF];    // V fp16, row-scaled
    alignas(1024) unsigned char Q[2][TF_HALF_BYTES];   // Q~ fp16 (from the preparation kernel)
    alignas(1024) unsigned char dA[2][TF_HALF_BYTES];  // dA fp16, row-scaled (TMA from the gate pass)
    float gq[kD], gk[kD];
    float dsinv[2][TF_BM];   // 2^-e of each dS row, by head number % 2
    float mdot[2][TF_BM];    // mean(dy gamma xhat) of each row (RMSNorm backward), by head % 2
    float dgq[4][kD];        // this CTA's d_gamma_q, one slice per epilogue warp
    float2 cs[TF_HALF][TF_BM];  // epilogue: (cos, sin) of each row's rotated pairs, per step
    uint64_t bar[QB_COUNT];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(BwdQTcSmem) + 1024 <= 227 * 1024, "query-major shared memory over the 227 KB a CTA may use");

// In-place fp16 conversion of a raw bf16 V tile by its 128 owner threads (thread r = row r;
// the four warps of one warpgroup, named barrier 1), with one power-of-two scale for the whole
// tile: the tile's max|v| lands in [2^13, 2^14).  (fp16 keeps its relative precision down to
// 2^-14, so one scale per tile loses nothing against one per row for any realistic spread of
// row magnitudes, and it makes the dP scale per tile instead of per key.)  Both backward
// kernels convert the same 128-row tiles the same way, so their fp16 V agree bit for bit.
// `red`: 4 floats of shared scratch; the caller alternates two so that the next tile does not
// overwrite values still being read.  Returns 2^-e; the row's 2-norm in *norm if wanted.
__device__ __forceinline__ float v_tile_to_f16(unsigned char* h0, unsigned char* h1, int r, float* red, float* norm) {
    float mx = 0.f, ss = 0.f;
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {
        const uint4 u = *tile_chunk(h0, h1, r, ch);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 t = unpack_bf16(w[e]);
            mx = fmaxf(mx, fmaxf(fabsf(t.x), fabsf(t.y)));
            ss = fmaf(t.x, t.x, fmaf(t.y, t.y, ss));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) red[(r >> 5) & 3] = mx;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const int e = fit_exp(mx);
    const float sc = ldexpf(1.0f, e);
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {
        uint4* pc = tile_chunk(h0, h1, r, ch);
        const uint4 u = *pc;
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 t = unpack_bf16(w[k]);
            w[k] = pack2<true>(t.x * sc, t.y * sc);
        }
        *pc = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (norm) *norm = sqrtf(ss);
    return ldexpf(1.0f, -e);
}

// =====================================================================  Q / K / V preparation

constexpr int KP_THREADS = 128;

template <bool IS_K>
struct PrepSmem {
    alignas(1024) unsigned char X[2][TF_HALF_BYTES];                 // raw k or q -> K~ / Q~ in place
    alignas(1024) unsigned char V[IS_K ? 2 : 1][IS_K ? TF_HALF_BYTES : 16];  // raw v -> fp16 in place
    float gq[kD], gk[kD];
    float vred[4];
    uint64_t bar;
};

// One CTA per 128-row tile (b, head, t): a key tile (IS_K: K~ and V) or a query tile (Q~).
// K~ = fp16(RoPE(gamma_k * k / rms) * oscale) and V * 2^e (one e per tile), or Q~ likewise
// from q and gamma_q, go to the workspace; the in-place conversion is the one the kernels
// once ran in their prologues (same device functions and angle values, same bits; the
// angles sit in registers here).  Also saved: each row's inverse RMS (RMSNorm backward of dq,
// dk), the raw norm of each v row (dS^T scale) and the V tile scale.  Several CTAs per SM keep
// tile loads, conversions and stores of different tiles in flight.
// WITH_K false (key tiles only): V alone, for a backward given the forward's K~ and inverse RMS.
// ANY: any number of rotated pairs, the angles formed as needed (else the layer's 21, in registers)
template <bool IS_K, bool WITH_K, bool ANY>
__device__ __forceinline__ void prep_tile(const BwdTcParams& p) {
    const LayerParams& L = p.P.L;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    PrepSmem<IS_K>& sm =
        *reinterpret_cast<PrepSmem<IS_K>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int r = threadIdx.x;
    // query tiles cover the query rows q_off .. S-1 (tile t at position q_off + 128 t; Q~ and
    // the inverse RMS are stored by position), key tiles every position
    const int nt = ((IS_K ? L.S : L.Sq) + TF_BN - 1) / TF_BN, x0 = IS_K ? 0 : L.q_off;
    const int H = IS_K ? L.Hkv : L.Hq;
    const int t = (int)blockIdx.x % nt, chain = (int)blockIdx.x / nt;
    const int h = chain % H, b = chain / H;
    volatile int abort = 0;
    if (r == 0) {
        mbar_init(&sm.bar, 1);
        fence_barrier_init();
    }
    sm.gq[r] = L.gamma_q[r];
    sm.gk[r] = L.gamma_k[r];
    __syncthreads();
    if (r == 0) {
        const CUtensorMap* src = IS_K ? &p.tm_k : &p.tm_q;
        mbar_expect_tx(&sm.bar, ((IS_K ? 1 : 0) + (WITH_K ? 1 : 0)) * TF_TILE_BYTES);
        if constexpr (WITH_K) {
            tma_load_4d(sm.X[0], src, &sm.bar, 0, h, t * TF_BN, b);
            tma_load_4d(sm.X[1], src, &sm.bar, 64, h, t * TF_BN, b);
        }
        if constexpr (IS_K) {
            tma_load_4d(sm.V[0], &p.tm_v, &sm.bar, 0, h, t * TF_BN, b);
            tma_load_4d(sm.V[1], &p.tm_v, &sm.bar, 64, h, t * TF_BN, b);
        }
    }
    const int pos = x0 + t * TF_BN + r;
    float2 csr[WITH_K && !ANY ? TF_HALF : 1];  // (cos, sin) of the rotated pairs at this row's position
    if constexpr (WITH_K && !ANY) {
#pragma unroll
        for (int q = 0; q < TF_HALF; ++q) rope_cs(L.theta[q], pos, csr[q].x, csr[q].y);
    }
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    // one decision for the whole CTA (the V conversion below has a CTA-wide barrier)
    const bool ok = __syncthreads_and(mbar_wait(&sm.bar, 0, &abort, 250)) != 0;
    if (ok) {
        float rinv = 0.f;
        if constexpr (WITH_K && ANY)
            rinv = tf_prologue_row_any<true>(sm.X[0], sm.X[1], r, IS_K ? sm.gk : sm.gq, L, pos, oscale);
        else if constexpr (WITH_K)
            rinv = tf_prologue_row_at<true>(sm.X[0], sm.X[1], r, IS_K ? sm.gk : sm.gq, L,
                                            [&](int q) { return csr[q]; }, oscale);
        const size_t ro = ((size_t)b * H + h) * L.S + pos;
        if constexpr (IS_K) {
            float vn = 0.f;
            const float vt = v_tile_to_f16(sm.V[0], sm.V[1], r, sm.vred, &vn);
            if (pos < L.S) {
                if constexpr (WITH_K) p.krinv[ro] = rinv;
                p.vnorm[ro] = vn;
            }
            if (r == 0) p.vtinv[(size_t)chain * nt + t] = vt;
        } else {
            if (pos < L.S) p.qrinv[ro] = rinv;
        }
        fence_proxy_async_smem();
    } else if (r == 0) {
        mbar_wait_drain(&sm.bar, 0);  // the loads must land before the CTA exits
    }
    __syncthreads();
    if (r == 0) {
        if (ok) {
            const CUtensorMap* dst = IS_K ? &p.tm_k16 : &p.tm_q16;
            if constexpr (WITH_K) {
                tma_store_4d(dst, sm.X[0], 0, h, x0 + t * TF_BN, b);
                tma_store_4d(dst, sm.X[1], 64, h, x0 + t * TF_BN, b);
            }
            if constexpr (IS_K) {
                tma_store_4d(&p.tm_v16, sm.V[0], 0, h, t * TF_BN, b);
                tma_store_4d(&p.tm_v16, sm.V[1], 64, h, t * TF_BN, b);
            }
            tma_store_commit();
            tma_store_wait_read();
        } else if (p.err) {
            atomicExch(p.err, 250);
        }
    }
}

template <bool ANY>
__global__ void __launch_bounds__(KP_THREADS, 3) bwd_prep_kv_kernel(const __grid_constant__ BwdTcParams p) {
    prep_tile<true, true, ANY>(p);
}
template <bool ANY>
__global__ void __launch_bounds__(KP_THREADS, 4) bwd_prep_q_kernel(const __grid_constant__ BwdTcParams p) {
    prep_tile<false, true, ANY>(p);
}
__global__ void __launch_bounds__(KP_THREADS, 3) bwd_prep_v_kernel(const __grid_constant__ BwdTcParams p) {
    prep_tile<true, false, false>(p);
}

// ANY: any number of rotated pairs in the dq epilogue (else the layer's 21, angles shared per step)
template <bool ANY>
__global__ void __launch_bounds__(TB_THREADS, 1) bwd_q_tc_kernel(const __grid_constant__ BwdTcParams p) {
    const LayerParams& L = p.P.L;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    BwdQTcSmem& sm = *reinterpret_cast<BwdQTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &sm.abort;
    const int G = L.G;
    const int t_begin = (int)(((long long)blockIdx.x * p.total) / gridDim.x);
    const int t_end = (int)(((long long)(blockIdx.x + 1) * p.total) / gridDim.x);

    if (tid == 0) {
        sm.abort = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.bar[QB_KFULL + i], 1);
            mbar_init(&sm.bar[QB_KEMPTY + i], 1);
            mbar_init(&sm.bar[QB_VFULL + i], 1);
            mbar_init(&sm.bar[QB_VEMPTY + i], 1);
        }
        mbar_init(&sm.bar[QB_QFULL], 1);
        mbar_init(&sm.bar[QB_QEMPTY], 1);
        mbar_init(&sm.bar[QB_DAEMPTY], 1);
        mbar_init(&sm.bar[QB_DAFULL], 1);
        mbar_init(&sm.bar[QB_DPFULL], 1);
        mbar_init(&sm.bar[QB_DSFULL], 128);
        mbar_init(&sm.bar[QB_DQFULL], 1);
        mbar_init(&sm.bar[QB_DQEMPTY], 128);
        mbar_init(&sm.bar[QB_DONE], 1);
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
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k);
        prefetch_tmap(&p.tm_v);
        prefetch_tmap(&p.tm_da);
        prefetch_tmap(&p.tm_k16);
        prefetch_tmap(&p.tm_v16);
        prefetch_tmap(&p.tm_q16);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // TMEM ping-pong over two 256-column halves, by head number m:
    //   S(m) -> half m%2, dP(m) -> the other half; dS(m) (fp16) over the first 128 columns of
    //   S(m) and dQ(m) in the last 128.  So S(m+1) can be issued as soon as dQ(m) is, while the
    //   epilogue still reads dQ(m); only dP(m+1) waits for that epilogue.
    auto tm_half = [&](int m) -> uint32_t { return tmem + 256u * (uint32_t)(m & 1); };
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    const float c2 = L.scale_log2 / (oscale * oscale);
    // mdot = scale / (D oscale^2) * sum_j dS_ij S_ij  (S as accumulated in TMEM)
    const float mdot_f = c2 * kLn2 / (float)kD;

    // Registers by warpgroup (4 x 128 in all, set at the top of each role): TMA / MMA issue
    // 72, softmax 176, idle 24, epilogue 240 (it holds a whole dq~ row so that it can release
    // TMEM before its arithmetic).  This split is the one without spills.
    if (warp < 4) {
        reg_dealloc<72>();
        if (warp == 0) {
            // ================================================ K / V producer
            if (lane == 0) {
                int n_next = 0;
                int last_k[2] = {-1, -1}, last_v[2] = {-1, -1};
                auto load_tile = [&](int n, int b, int kvh, int kt) -> bool {
                    const int slot = n & 1;
                    if (n >= 2 && !mbar_wait(&sm.bar[QB_KEMPTY + slot], ((n >> 1) - 1) & 1, abort, 101)) return false;
                    mbar_expect_tx(&sm.bar[QB_KFULL + slot], TF_TILE_BYTES);
                    tma_load_4d(sm.K[0] + slot * TF_HALF_BYTES, &p.tm_k16, &sm.bar[QB_KFULL + slot], 0, kvh, kt * TF_BN, b);
                    tma_load_4d(sm.K[1] + slot * TF_HALF_BYTES, &p.tm_k16, &sm.bar[QB_KFULL + slot], 64, kvh, kt * TF_BN, b);
                    last_k[slot] = n;
                    if (n >= 2 && !mbar_wait(&sm.bar[QB_VEMPTY + slot], ((n >> 1) - 1) & 1, abort, 102)) return false;
                    mbar_expect_tx(&sm.bar[QB_VFULL + slot], TF_TILE_BYTES);
                    tma_load_4d(sm.V[0] + slot * TF_HALF_BYTES, &p.tm_v16, &sm.bar[QB_VFULL + slot], 0, kvh, kt * TF_BN, b);
                    tma_load_4d(sm.V[1] + slot * TF_HALF_BYTES, &p.tm_v16, &sm.bar[QB_VFULL + slot], 64, kvh, kt * TF_BN, b);
                    last_v[slot] = n;
                    return true;
                };
                for (int t = t_begin; t < t_end && !*abort; ++t) {
                    const StepInfo st = decode_step(L, t, t_begin, t_end);
                    if (st.fresh && !load_tile(n_next++, st.b, st.kvh, st.qb - 1)) break;
                    if (!load_tile(n_next++, st.b, st.kvh, st.qb)) break;
                }
                for (int slot = 0; slot < 2; ++slot) {
                    if (last_k[slot] >= 0) mbar_wait_drain(&sm.bar[QB_KFULL + slot], (last_k[slot] >> 1) & 1);
                    if (last_v[slot] >= 0) mbar_wait_drain(&sm.bar[QB_VFULL + slot], (last_v[slot] >> 1) & 1);
                }
            }
        } else if (warp == 2) {
            // ================================================ Q and dA producer (single buffers)
            if (lane == 0) {
                int m = 0, last = -1, last_da = -1;
                bool ok = true;
                for (int t = t_begin; t < t_end && ok && !*abort; ++t) {
                    const StepInfo st = decode_step(L, t, t_begin, t_end);
                    for (int h = 0; h < G; ++h, ++m) {
                        const int hg = st.kvh * G + h;
                        if (m >= 1 && !(ok = mbar_wait(&sm.bar[QB_QEMPTY], (m - 1) & 1, abort, 103))) break;
                        mbar_expect_tx(&sm.bar[QB_QFULL], TF_TILE_BYTES);
                        tma_load_4d(sm.Q[0], &p.tm_q16, &sm.bar[QB_QFULL], 0, hg, st.qb * TF_BM, st.b);
                        tma_load_4d(sm.Q[1], &p.tm_q16, &sm.bar[QB_QFULL], 64, hg, st.qb * TF_BM, st.b);
                        last = m;
                        if (m >= 1 && !(ok = mbar_wait(&sm.bar[QB_DAEMPTY], (m - 1) & 1, abort, 104))) break;
                        mbar_expect_tx(&sm.bar[QB_DAFULL], TF_TILE_BYTES);
                        tma_load_4d(sm.dA[0], &p.tm_da, &sm.bar[QB_DAFULL], 0, hg, st.qb * TF_BM, st.b);
                        tma_load_4d(sm.dA[1], &p.tm_da, &sm.bar[QB_DAFULL], 64, hg, st.qb * TF_BM, st.b);
                        last_da = m;
                    }
                }
                if (last >= 0) mbar_wait_drain(&sm.bar[QB_QFULL], last & 1);
                if (last_da >= 0) mbar_wait_drain(&sm.bar[QB_DAFULL], last_da & 1);
            }
        } else if (warp == 1) {
            // ================================================ MMA issuer
            if (lane == 0) {
                constexpr uint32_t IDESC_N256 = idesc_f16(128, 256, false);
                constexpr uint32_t IDESC_DQ = idesc_f16(128, 128, true);
                const uint32_t q_base = smem_u32(sm.Q[0]), da_base = smem_u32(sm.dA[0]);
                const uint32_t k_base = smem_u32(sm.K[0]), v_base = smem_u32(sm.V[0]);
                int n_next = 0, n_prev = 0, n_cur = 0, m = 0;
                bool ok = true;
                for (int t = t_begin; t < t_end && ok; ++t) {
                    const StepInfo st = decode_step(L, t, t_begin, t_end);
                    if (st.fresh) {
                        n_prev = n_next++;
                        n_cur = n_next++;
                        ok = mbar_wait(&sm.bar[QB_KFULL + (n_prev & 1)], (n_prev >> 1) & 1, abort, 110) &&
                             mbar_wait(&sm.bar[QB_VFULL + (n_prev & 1)], (n_prev >> 1) & 1, abort, 111);
                    } else {
                        n_prev = n_cur;
                        n_cur = n_next++;
                    }
                    ok = ok && mbar_wait(&sm.bar[QB_KFULL + (n_cur & 1)], (n_cur >> 1) & 1, abort, 112) &&
                         mbar_wait(&sm.bar[QB_VFULL + (n_cur & 1)], (n_cur >> 1) & 1, abort, 113);
                    for (int h = 0; h < G && ok; ++h, ++m) {
                        const uint32_t tA = tm_half(m), tB = tm_half(m + 1);
                        if (!(ok = mbar_wait(&sm.bar[QB_QFULL], m & 1, abort, 114))) break;
                        if (!(ok = mbar_wait(&sm.bar[QB_DAFULL], m & 1, abort, 118))) break;
                        // dP(m) goes to tB once the epilogue of head m-1 has read dQ(m-1) there
                        if (m >= 1 && !(ok = mbar_wait(&sm.bar[QB_DQEMPTY], (m - 1) & 1, abort, 115))) break;
                        tc_fence_after();
                        // S = Q~ K~^T -> tA (its columns were last read by the softmax of head m-1, as
                        // dP, and by the epilogue of head m-2) and dP = dA V^T -> tB, K-step by
                        // K-step in turn: two independent accumulation chains overlap in the pipe
    #pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t half = kk >> 2, within = (kk & 3) * 32;
                            const uint64_t aq = sdesc_sw128(q_base + half * TF_HALF_BYTES + within, 16, 1024);
                            const uint64_t bk = sdesc_sw128(k_base + half * TF_RING_HALF + within, 16, 1024);
                            mma_ss(tA, aq, bk, IDESC_N256, kk > 0 ? 1u : 0u);
                            const uint64_t ad = sdesc_sw128(da_base + half * TF_HALF_BYTES + within, 16, 1024);
                            const uint64_t bv = sdesc_sw128(v_base + half * TF_RING_HALF + within, 16, 1024);
                            mma_ss(tB, ad, bv, IDESC_N256, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&sm.bar[QB_QEMPTY]);
                        mma_commit(&sm.bar[QB_DAEMPTY]);
                        mma_commit(&sm.bar[QB_DPFULL]);
                        if (h == G - 1) {
                            mma_commit(&sm.bar[QB_VEMPTY + (n_prev & 1)]);
                            if (st.release_cur) mma_commit(&sm.bar[QB_VEMPTY + (n_cur & 1)]);
                        }
                        if (!(ok = mbar_wait(&sm.bar[QB_DSFULL], m & 1, abort, 116))) break;
                        tc_fence_after();
                        // dQ~ = dS K~ -> tA + 128 : dS fp16 in tA (16 keys = 8 columns per step), K~ MN-major
    #pragma unroll
                        for (int kk = 0; kk < 16; ++kk) {
                            const uint64_t bk = sdesc_sw128(k_base + kk * 16 * 128, TF_RING_HALF, 1024);
                            mma_ts(tA + 128, tA + kk * 8, bk, IDESC_DQ, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&sm.bar[QB_DQFULL]);
                        if (h == G - 1) {
                            mma_commit(&sm.bar[QB_KEMPTY + (n_prev & 1)]);
                            if (st.release_cur) mma_commit(&sm.bar[QB_KEMPTY + (n_cur & 1)]);
                        }
                    }
                }
                mma_commit(&sm.bar[QB_DONE]);
                mbar_wait(&sm.bar[QB_DONE], 0, abort, 117);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        reg_alloc<176>();
        // ================================================ Delta, dS (thread = query row)
        const int r = tid - 128, wq = warp - 4;
        const int nkt = (L.S + TF_BN - 1) / TF_BN, Spad = row_stride(L.S);
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        int n_next = 0, n_cur = 0, m = 0;
        for (int t = t_begin; t < t_end; ++t) {
            const StepInfo st = decode_step(L, t, t_begin, t_end);
            if (st.fresh) n_next++;  // the previous tile takes a ring slot of its own
            n_cur = n_next++;
            const int q0 = st.qb * TF_BM, i = q0 + r;
            const int slot_cur = n_cur & 1;
            const int base0 = (slot_cur == 0 ? q0 : q0 - TF_BN), base1 = (slot_cur == 1 ? q0 : q0 - TF_BN);
            // V tile scales of the two ring slots (a tile before the sequence start holds no key)
            const float* vtrow = p.vtinv + ((size_t)st.b * L.Hkv + st.kvh) * nkt;
            const float vt0 = base0 >= 0 ? vtrow[base0 / TF_BN] : 0.f, vt1 = base1 >= 0 ? vtrow[base1 / TF_BN] : 0.f;
            const int imin = q0 + 32 * wq, imax = imin + 31;
            // chunk c8 (32 keys from kp0) against this warp's 32 rows: live = some pair visible,
            // full = every pair visible (warp-uniform; masks skipped)
            auto chunk_kp0 = [&](int c8) { return (c8 < 4 ? base0 : base1) + (c8 & 3) * 32; };
            auto chunk_live = [&](int kp0) {
                return imin < L.S && kp0 <= imax && kp0 + 31 > imin - L.W && kp0 + 31 >= 0 && kp0 < L.S;
            };
            auto chunk_full = [&](int kp0) {
                return kp0 + 31 <= imin && kp0 > imax - L.W && kp0 >= 0 && kp0 + 31 < L.S;
            };
            bool stop = false;
            for (int h = 0; h < G; ++h, ++m) {
                const int hg = st.kvh * G + h;
                const size_t ro = ((size_t)st.b * L.Hq + hg) * L.S + (i < L.S ? i : 0);
                const size_t rp = ((size_t)st.b * L.Hq + hg) * Spad + i;  // padded row arrays
                // the forward's log-sum-exp (base 2): its scores are these, bit for bit
                const float lse2 = i < L.S ? p.P.lse[ro] * kLog2e : INFINITY;
                const float dai = i < L.S ? p.dainv[rp] : 0.f;  // undoes the dA row scale
                const uint32_t tS = tm_half(m) + lane_off, tP = tm_half(m + 1) + lane_off;
                if (!mbar_wait(&sm.bar[QB_DPFULL], m & 1, abort, 121)) { stop = true; break; }
                tc_fence_after();
                const float kd0 = dai * vt0, kd1 = dai * vt1;
                // pass 1: P = 2^(S c2 - lse), P dP (written back over S and dP), Delta = sum P dP,
                // max |P dP|, and the RMSNorm backward's row sums  a = sum P dP S,  b = sum P S
                float num = 0.f, mpd = 0.f, sa = 0.f, sb = 0.f;
                const int klo = max(i - L.W + 1, 0), khi = min(i, L.S - 1);  // this row's visible keys
#pragma unroll 1
                for (int c8 = 0; c8 < 8; ++c8) {
                    const int kp0 = chunk_kp0(c8);
                    if (!chunk_live(kp0)) continue;
                    float sv[32], dv[32];
                    tmem_ld32f(tS + 32 * c8, sv);
                    tmem_ld32f(tP + 32 * c8, dv);
                    tmem_wait_ld();
                    float cnum = 0.f, cmpd = 0.f, csa = 0.f;
                    if (chunk_full(kp0))
                        q_pass1_chunk<true>(sv, dv, 0u, c2, lse2, cnum, cmpd, csa, sb);
                    else
                        q_pass1_chunk<false>(sv, dv, bit_range(klo - kp0, khi - kp0), c2, lse2, cnum, cmpd, csa, sb);
                    const float kd = c8 < 4 ? kd0 : kd1;  // dP = dv * kd on this key tile
                    num = fmaf(kd, cnum, num);
                    mpd = fmaxf(mpd, fabsf(kd) * cmpd);
                    sa = fmaf(kd, csa, sa);
                    tmem_st32f(tS + 32 * c8, sv);
                    tmem_st32f(tP + 32 * c8, dv);
                }
                tmem_wait_st();
                const float delta = num;
                // |dS| = |P dP - P Delta| <= max |P dP| + |Delta|
                const float dsc = ldexpf(1.0f, fit_exp(mpd + fabsf(delta)));
                // pass 2: dS = (P dP - P Delta) dsc, fp16, over the first 128 columns of S
#pragma unroll 1
                for (int c8 = 0; c8 < 8; ++c8) {
                    const int kp0 = chunk_kp0(c8);
                    uint32_t pk[16];
                    if (chunk_live(kp0)) {
                        float pv[32], pd[32];
                        tmem_ld32f(tS + 32 * c8, pv);
                        tmem_ld32f(tP + 32 * c8, pd);
                        tmem_wait_ld();
                        // pd holds P dv: dS dsc = P dv (kd dsc) - P (Delta dsc)
                        const float ka = (c8 < 4 ? kd0 : kd1) * dsc, kb = -delta * dsc;
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
                    tmem_st16(tS + 16 * c8, pk);
                }
                tmem_wait_st();
                if (i < Spad) {
                    // Delta and the base-2 lse per row for the key-major kernel; past S the
                    // neutral values (P = 0 there, and the dA scale 0)
                    p.P.delta[rp] = i < L.S ? delta : 0.f;
                    p.lse2p[rp] = lse2;
                    if (i >= L.S) p.dainv[rp] = 0.f;
                }
                sm.dsinv[m & 1][r] = 1.0f / dsc;
                sm.mdot[m & 1][r] = fmaf(-delta, sb, sa) * mdot_f;  // sum dS S = a - Delta b
                tc_fence_before();
                mbar_arrive(&sm.bar[QB_DSFULL]);
            }
            if (stop) break;
        }
    } else if (warp >= 8 && warp < 12) {
        // (no prologue: Q~, K~ and V arrive converted from the preparation kernel; the
        // warpgroup only hands its registers to the others)
        reg_dealloc<24>();
    } else if (warp >= 12) {
        reg_alloc<240>();
        // ================================================ dq epilogue (thread = query row)
        const int r = tid - 384, wq = warp - 12;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        int m = 0;
        bool ok = true;
        for (int t = t_begin; t < t_end && ok; ++t) {
            const StepInfo st = decode_step(L, t, t_begin, t_end);
            const int i = st.qb * TF_BM + r;
            const bool valid = i < L.S;
            // the row's rotation angles, shared by the G heads of the step (own column only)
#pragma unroll 1
            for (int q = 0; !ANY && q < TF_HALF; ++q) rope_cs(L.theta[q], i, sm.cs[q][r].x, sm.cs[q][r].y);
            for (int h = 0; h < G; ++h, ++m) {
                const int hg = st.kvh * G + h;
                const size_t off = ((size_t)(st.b * (size_t)L.S + (valid ? i : 0)) * L.Hq + hg) * kD;
                const float rinv = valid ? p.qrinv[((size_t)st.b * L.Hq + hg) * L.S + i] : 0.f;
                uint4 xv0[8];  // first half of the raw q row, in flight during the wait
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    xv0[c] = valid ? __ldg(reinterpret_cast<const uint4*>(L.q + off) + c) : make_uint4(0u, 0u, 0u, 0u);
                if (!(ok = mbar_wait(&sm.bar[QB_DQFULL], m & 1, abort, 140))) break;
                tc_fence_after();
                float dy[128];
                const uint32_t tq = tm_half(m) + 128 + lane_off;
                tmem_ld32f(tq, dy);
                tmem_ld32f(tq + 32, dy + 32);
                tmem_ld32f(tq + 64, dy + 64);
                tmem_ld32f(tq + 96, dy + 96);
                tmem_wait_ld();
                const float f = L.scale * sm.dsinv[m & 1][r] / oscale;
                const float mdot = sm.mdot[m & 1][r];
                tc_fence_before();
                mbar_arrive(&sm.bar[QB_DQEMPTY]);  // dQ(m) is in registers: TMEM free for dP(m+1)
                if constexpr (ANY)
                    row_rope_rms_backward_regs<0>(dy, f, mdot, rinv, xv0, L.q + off, p.P.dq + off, valid, i, sm.gq,
                                                  sm.dgq[wq], L);
                else
                    row_rope_rms_backward_cs(dy, f, mdot, rinv, xv0, L.q + off, p.P.dq + off, valid,
                                             [&](int q) { return sm.cs[q][r]; }, sm.gq, sm.dgq[wq]);
            }
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

// =====================================================================  key-major kernel

constexpr int KV_SLOTS = 4;                      // Q~ / dA ring depth, in 64-query halves
constexpr uint32_t KV_SLOT_HALF = 64u * 128u;   // 64 rows x 128 bytes: one d-half of a slot

enum KBar {
    KB_KVFULL = 0, KB_KVEMPTY = 2,
    KB_QFULL = 3, KB_QEMPTY = 11,  // by ring slot (KV_SLOTS each)
    KB_SFULL = 15, KB_PFULL = 17,                 // by TMEM buffer (2 each)
    KB_DVKFULL = 19, KB_DVKEMPTY = 20, KB_DONE = 21, KB_RED = 22,
    KB_STATS = 23,  // a unit's scales are in shared memory; by unit number % 2
    KB_DVKDONE = 25,  // the dV / dK products of a half have read their TMEM buffer; by buffer (2)
    KB_COUNT = 27
};

struct BwdKTcSmem {
    alignas(1024) unsigned char K[2][TF_HALF_BYTES];      // K~ fp16 of the unit's key tile
    alignas(1024) unsigned char V[2][TF_HALF_BYTES];      // V fp16, row-scaled
    // ring of KV_SLOTS slots, one per 64-query half: Q~ and dA rows of the half, each as two
    // d-halves of 64 rows x 128 bytes (the SW128 layout of a 64-row TMA box)
    alignas(1024) unsigned char Q[KV_SLOTS][2][KV_SLOT_HALF];
    alignas(1024) unsigned char dA[KV_SLOTS][2][KV_SLOT_HALF];
    float gq[kD], gk[kD];
    // per query column of the slot, loaded by TMA with the slot's rows (neutral values past
    // the sequence end, where every pair is masked): the forward's lse in base 2, Delta, 2^-e
    // of the dA row
    alignas(128) float lsec[KV_SLOTS][64];
    alignas(128) float delta[KV_SLOTS][64];
    alignas(128) float dcol[KV_SLOTS][64];
    float vtinv[4];          // 2^-e of the unit's V tile, by unit number % 4
    float dsc[4][TF_BN];     // 2^e of each dS^T row, by unit number % 4
    // 4 deep: the prologue writes a unit's scales at its start, while the epilogue of an earlier
    // unit may still read its own (with one query head per KV head a unit has two iterations)
    float uinv[4];           // 2^-E, E = the unit's smallest dA row exponent, by unit number % 4
    float kmdot[2][2][TF_BN];  // mean(dy gamma xhat) of each key row (RMSNorm backward): the two
                               // softmax warpgroups' shares, by unit parity
    float red[2][2][4];      // per-warp maxima for the unit statistics, by call parity
    float dgk[4][kD];        // this CTA's d_gamma_k, one slice per epilogue warp
    uint64_t bar[KB_COUNT];
    uint32_t tmem_base;
    int abort;
};

struct UnitInfo {
    int b, kvh, kt, nit;   // nit = iterations: heads x query blocks that see the key tile
    int qb0;               // the first of those query blocks
};
// Unit u: key tile kt of (b, KV head).  Sliding windows (W <= 128) sweep the units of a chain
// in order (u = chain * tiles + kt), and query blocks kt and kt + 1 see the tile; wide windows
// run one unit per CTA, heaviest (first tiles) first (u = kt * chains + chain), and the
// query blocks that see tile kt run from kt (or the block of the first query row, q_off / 128,
// if later) to the block of the last query whose window reaches the tile's last key,
// kt*128 + 127 + W - 1.  With q_off > 0 the tiles before wide_first_tile(L) have no query at
// all: they take no unit (the launcher zeroes their dk and dv).
__device__ __forceinline__ UnitInfo decode_unit(const LayerParams& L, int u, bool wide) {
    const int nkb = (L.S + TF_BN - 1) / TF_BN;
    UnitInfo x;
    int chain;
    if (wide) {
        const int chains = L.B * L.Hkv;
        x.kt = wide_first_tile(L) + u / chains;
        chain = u % chains;
        // W <= S here (the launcher clamps it), so the sum stays in range
        const int last_q = x.kt * TF_BN + TF_BN - 1 + L.W - 1;
        const int qb_hi = min(nkb - 1, last_q / TF_BM);
        x.qb0 = max(x.kt, L.q_off / TF_BM);
        x.nit = L.G * (qb_hi - x.qb0 + 1);
    } else {
        chain = u / nkb;
        x.kt = u - chain * nkb;
        x.qb0 = x.kt;
        x.nit = L.G * ((x.kt + 1 < nkb) ? 2 : 1);  // W <= 128: blocks kt and kt + 1
    }
    x.b = chain / L.Hkv;
    x.kvh = chain - x.b * L.Hkv;
    return x;
}
// iteration it of a unit: query block qb0 + it / G, head it % G
__device__ __forceinline__ void decode_iter(const LayerParams& L, const UnitInfo& x, int it, int& qb, int& hg) {
    qb = x.qb0 + it / L.G;
    hg = x.kvh * L.G + it % L.G;
}

template <bool WIDE, bool ANY>
__global__ void __launch_bounds__(TB_THREADS, 1) bwd_kv_tc_kernel(const __grid_constant__ BwdTcParams p) {
    const LayerParams& L = p.P.L;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    BwdKTcSmem& sm = *reinterpret_cast<BwdKTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort = &sm.abort;
    const int u_begin = (int)(((long long)blockIdx.x * p.total) / gridDim.x);
    const int u_end = (int)(((long long)(blockIdx.x + 1) * p.total) / gridDim.x);

    if (tid == 0) {
        sm.abort = 0;
        mbar_init(&sm.bar[KB_KVFULL], 1);
        mbar_init(&sm.bar[KB_KVEMPTY], 1);
        for (int i = 0; i < KV_SLOTS; ++i) {
            mbar_init(&sm.bar[KB_QFULL + i], 1);
            mbar_init(&sm.bar[KB_QEMPTY + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.bar[KB_SFULL + i], 1);
            mbar_init(&sm.bar[KB_PFULL + i], 128);
        }
        mbar_init(&sm.bar[KB_DVKFULL], 1);
        mbar_init(&sm.bar[KB_DVKEMPTY], 128);
        mbar_init(&sm.bar[KB_DONE], 2);  // both MMA issuers
        mbar_init(&sm.bar[KB_DVKDONE], 1);
        mbar_init(&sm.bar[KB_DVKDONE + 1], 1);
        mbar_init(&sm.bar[KB_RED], 4);  // one arrival per epilogue warp
        mbar_init(&sm.bar[KB_STATS], 128);
        mbar_init(&sm.bar[KB_STATS + 1], 128);
        fence_barrier_init();
    }
    if (tid < kD) {
        sm.gq[tid] = L.gamma_q[tid];
        sm.gk[tid] = L.gamma_k[tid];
        for (int w = 0; w < 4; ++w) sm.dgk[w][tid] = 0.f;
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k);
        prefetch_tmap(&p.tm_v);
        prefetch_tmap(&p.tm_da);
        prefetch_tmap(&p.tm_k16);
        prefetch_tmap(&p.tm_v16);
        prefetch_tmap(&p.tm_q16);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // TMEM: two 128-column buffers, one per 64-query half of an iteration: S^T in columns
    // [0,64) and dP^T in [64,128) of the buffer, P^T and dS^T (fp16) over their first 32;
    // dV and dK accumulators in [256,384) and [384,512).
    const uint32_t TM_DV = tmem + 256,
                   TM_DK = tmem + 384;
    const float oscale = qk_fp16_scale(sm.gq, sm.gk);
    const float c2 = L.scale_log2 / (oscale * oscale);
    const float mdot_f = c2 * kLn2 / (float)kD;  // scale / (D oscale^2)

    // Registers by warpgroup (4 x 128 in all, set at the top of each role): TMA / MMA issue
    // 64, the two softmax warpgroups 128 each, epilogue 192 (it holds a whole dk~ row so that
    // it can release TMEM before its arithmetic).
    if (warp < 4) {
        reg_dealloc<64>();
        if (warp == 0) {
            // ================================================ TMA producer: K, V per unit; Q~, dA per 64-query half
            if (lane == 0) {
                int hs = 0, uu = 0, last_q[KV_SLOTS];
                for (int i = 0; i < KV_SLOTS; ++i) last_q[i] = -1;
                auto load_kv = [&](const UnitInfo& x) {
                    mbar_expect_tx(&sm.bar[KB_KVFULL], 2 * TF_TILE_BYTES);
                    tma_load_4d(sm.K[0], &p.tm_k16, &sm.bar[KB_KVFULL], 0, x.kvh, x.kt * TF_BN, x.b);
                    tma_load_4d(sm.K[1], &p.tm_k16, &sm.bar[KB_KVFULL], 64, x.kvh, x.kt * TF_BN, x.b);
                    tma_load_4d(sm.V[0], &p.tm_v16, &sm.bar[KB_KVFULL], 0, x.kvh, x.kt * TF_BN, x.b);
                    tma_load_4d(sm.V[1], &p.tm_v16, &sm.bar[KB_KVFULL], 64, x.kvh, x.kt * TF_BN, x.b);
                };
                bool ok = true;
                for (int u = u_begin; u < u_end && ok && !*abort; ++u, ++uu) {
                    const UnitInfo x = decode_unit(L, u, WIDE);
                    for (int it = 0; it < x.nit && ok; ++it) {
                        int qb, hg;
                        decode_iter(L, x, it, qb, hg);
                        for (int half = 0; half < 2; ++half, ++hs) {
                            const int slot = hs % KV_SLOTS;
                            if (hs >= KV_SLOTS &&
                                !(ok = mbar_wait(&sm.bar[KB_QEMPTY + slot], ((hs / KV_SLOTS) - 1) & 1, abort, 202)))
                                break;
                            const int row = qb * TF_BM + 64 * half;
                            mbar_expect_tx(&sm.bar[KB_QFULL + slot], 4 * KV_SLOT_HALF + 3 * 64 * 4);
                            tma_load_3d(sm.lsec[slot], &p.tm_lse, &sm.bar[KB_QFULL + slot], row, hg, x.b);  // base-2 lse
                            tma_load_3d(sm.delta[slot], &p.tm_delta, &sm.bar[KB_QFULL + slot], row, hg, x.b);
                            tma_load_3d(sm.dcol[slot], &p.tm_dainv, &sm.bar[KB_QFULL + slot], row, hg, x.b);
                            tma_load_4d(sm.Q[slot][0], &p.tm_q16h, &sm.bar[KB_QFULL + slot], 0, hg, row, x.b);
                            tma_load_4d(sm.Q[slot][1], &p.tm_q16h, &sm.bar[KB_QFULL + slot], 64, hg, row, x.b);
                            tma_load_4d(sm.dA[slot][0], &p.tm_dah, &sm.bar[KB_QFULL + slot], 0, hg, row, x.b);
                            tma_load_4d(sm.dA[slot][1], &p.tm_dah, &sm.bar[KB_QFULL + slot], 64, hg, row, x.b);
                            last_q[slot] = hs;
                            if (it == 0 && half == 0) {
                                // K, V of the unit once the previous unit's products are done; the
                                // unit's first query half went out before, as soon as its slot was free
                                if (uu >= 1 && !(ok = mbar_wait(&sm.bar[KB_KVEMPTY], (uu - 1) & 1, abort, 201))) break;
                                load_kv(x);
                            }
                        }
                    }
                }
                if (uu >= 1) mbar_wait_drain(&sm.bar[KB_KVFULL], (uu - 1) & 1);
                for (int i = 0; i < KV_SLOTS; ++i)
                    if (last_q[i] >= 0) mbar_wait_drain(&sm.bar[KB_QFULL + i], (last_q[i] / KV_SLOTS) & 1);
            }
        } else if (warp == 1 || warp == 2) {
            // ================================================ MMA issuers
            // Per 64-query half h (sweep order: unit, iteration, half), into TMEM buffer h % 2:
            //   S(h):   S^T = K~ Q~_h^T, dP^T = V dA_h^T      (M = 128 keys, N = 64, K = d)
            //   DVK(h): dV += P^T_h dA_h, dK~ += dS^T_h Q~_h  (K = 64 queries)
            // warp 1 issues the S products, warp 2 the DVK ones, so that neither thread's waits
            // and bookkeeping leave the tensor pipe without instructions: S(h+2) waits for
            // DVK(h) to have read buffer h % 2 (KB_DVKDONE), DVK(h) for the softmax of half h.
            if (lane == 0) {
                constexpr uint32_t IDESC_S = idesc_f16(128, 64, false);
                constexpr uint32_t IDESC_MN = idesc_f16(128, 128, true);
                // descriptors of each operand's first step; the others are offsets from them
                const uint64_t k_d = sdesc_sw128(smem_u32(sm.K[0]), 16, 1024);
                const uint64_t v_d = sdesc_sw128(smem_u32(sm.V[0]), 16, 1024);
                const uint64_t q_d = sdesc_sw128(smem_u32(sm.Q[0][0]), 16, 1024);
                const uint64_t da_d = sdesc_sw128(smem_u32(sm.dA[0][0]), 16, 1024);
                const uint64_t q_mn = sdesc_sw128(smem_u32(sm.Q[0][0]), KV_SLOT_HALF, 1024);
                const uint64_t da_mn = sdesc_sw128(smem_u32(sm.dA[0][0]), KV_SLOT_HALF, 1024);
                struct Cursor {
                    int u, uu, it, it_all, half;
                    UnitInfo x;
                    bool valid;
                };
                auto cur_first = [&]() {
                    Cursor c{u_begin, 0, 0, 0, 0, UnitInfo{}, u_begin < u_end};
                    if (c.valid) c.x = decode_unit(L, c.u, WIDE);
                    return c;
                };
                auto cur_next = [&](Cursor& c) {
                    if (++c.half < 2) return;
                    c.half = 0;
                    ++c.it_all;
                    if (++c.it < c.x.nit) return;
                    c.it = 0;
                    ++c.uu;
                    if (++c.u < u_end) c.x = decode_unit(L, c.u, WIDE);
                    else c.valid = false;
                };
                auto last_of_unit = [](const Cursor& c) { return c.half == 1 && c.it == c.x.nit - 1; };
                auto issue_s = [&](const Cursor& c) -> bool {
                    const int hs = 2 * c.it_all + c.half, slot = hs % KV_SLOTS;
                    if (c.it == 0 && c.half == 0 && !mbar_wait(&sm.bar[KB_KVFULL], c.uu & 1, abort, 210)) return false;
                    if (!mbar_wait(&sm.bar[KB_QFULL + slot], (hs / KV_SLOTS) & 1, abort, 211)) return false;
                    tc_fence_after();
                    const uint32_t tX = tmem + 128u * (uint32_t)c.half;
                    const uint32_t so = (uint32_t)slot * 2u * KV_SLOT_HALF;
                    // S^T and dP^T step by step in turn: two independent accumulation chains keep the
                    // tensor pipe busy where one dependent chain waits on each step
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t dh = kk >> 2, within = (kk & 3) * 32;
                        mma_ss(tX, sdesc_step(k_d, dh * TF_HALF_BYTES + within),
                               sdesc_step(q_d, so + dh * KV_SLOT_HALF + within), IDESC_S, kk > 0 ? 1u : 0u);
                        mma_ss(tX + 64, sdesc_step(v_d, dh * TF_HALF_BYTES + within),
                               sdesc_step(da_d, so + dh * KV_SLOT_HALF + within), IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sm.bar[KB_SFULL + c.half]);
                    if (last_of_unit(c)) mma_commit(&sm.bar[KB_KVEMPTY]);  // K, V read for the last time
                    return true;
                };
                auto issue_dvk = [&](const Cursor& c) -> bool {
                    const int hs = 2 * c.it_all + c.half, slot = hs % KV_SLOTS;
                    if (!mbar_wait(&sm.bar[KB_PFULL + c.half], c.it_all & 1, abort, 212)) return false;
                    if (c.it == 0 && c.half == 0 && c.uu >= 1 &&
                        !mbar_wait(&sm.bar[KB_DVKEMPTY], (c.uu - 1) & 1, abort, 213))
                        return false;
                    tc_fence_after();
                    const uint32_t tX = tmem + 128u * (uint32_t)c.half;
                    const uint32_t so = (uint32_t)slot * 2u * KV_SLOT_HALF;
                    const bool first = c.it == 0 && c.half == 0;
                    // A from TMEM (16 queries = 8 columns per step); B = dA / Q~ MN-major (N = d)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {  // dV and dK step by step in turn
                        mma_ts(TM_DV, tX + kk * 8, sdesc_step(da_mn, so + kk * 16 * 128), IDESC_MN,
                               (!first || kk > 0) ? 1u : 0u);
                        mma_ts(TM_DK, tX + 64 + kk * 8, sdesc_step(q_mn, so + kk * 16 * 128), IDESC_MN,
                               (!first || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&sm.bar[KB_QEMPTY + slot]);  // the half's Q~ and dA rows were read for the last time
                    mma_commit(&sm.bar[KB_DVKDONE + c.half]);  // TMEM buffer h % 2 read: free for S(h+2)
                    if (last_of_unit(c)) mma_commit(&sm.bar[KB_DVKFULL]);
                    return true;
                };
                bool ok = true;
                if (warp == 1) {
                    Cursor cs_ = cur_first();
                    for (int hs = 0; ok && cs_.valid; ++hs) {
                        if (hs >= 2 && !(ok = mbar_wait(&sm.bar[KB_DVKDONE + (hs & 1)], ((hs >> 1) - 1) & 1, abort, 215)))
                            break;
                        ok = issue_s(cs_);
                        cur_next(cs_);
                    }
                } else {
                    Cursor cd = cur_first();
                    while (ok && cd.valid) {
                        ok = issue_dvk(cd);
                        cur_next(cd);
                    }
                }
                mma_commit(&sm.bar[KB_DONE]);  // this thread's products, all complete before teardown
                mbar_wait(&sm.bar[KB_DONE], 0, abort, 214);
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // ================================================ P^T, dS^T (thread = key row)
        // Two warpgroups: warps 4-7 take the first 64-query half of every iteration (TMEM
        // buffer 0), warps 8-11 the second (buffer 1), so the halves' softmax runs in parallel.
        const int r = (tid - 128) & 127, wq = warp & 3, my_half = warp >= 8 ? 1 : 0;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        int it_all = 0, uu = 0;
        bool ok = true;
        for (int u = u_begin; u < u_end && ok; ++u, ++uu) {
            const UnitInfo x = decode_unit(L, u, WIDE);
            const int j = x.kt * TF_BN + r;
            float vin = 0.f, su = 0.f, dsc = 0.f;
            float kacc = 0.f;  // sum over the unit of dS^T S^T (unscaled dS^T): dk's RMSNorm row term
            for (int it = 0; it < x.nit && ok; ++it, ++it_all) {
                int qb, hg;
                decode_iter(L, x, it, qb, hg);
                const int q0 = qb * TF_BM;
                const int jmin = x.kt * TF_BN + 32 * wq, jmax = jmin + 31;
                for (int half = my_half; half == my_half && ok; ++half) {
                    const int hs = 2 * it_all + half, slot = hs % KV_SLOTS;
                    if (it == 0) {
                        if (!(ok = mbar_wait(&sm.bar[KB_STATS + (uu & 1)], (uu >> 1) & 1, abort, 223))) break;
                        vin = sm.vtinv[uu & 3];        // undoes the V tile scale of dP^T
                        su = 1.0f / sm.uinv[uu & 3];   // 2^E: P^T columns carry 2^(E - e_i)
                        dsc = sm.dsc[uu & 3][r];
                    }
                    // 64-query half in TMEM buffer `half`: S^T at columns [0,64), dP^T at [64,128);
                    // its S MMA waited for the slot's TMA, per-column values included
                    if (!(ok = mbar_wait(&sm.bar[KB_SFULL + half], it_all & 1, abort, 222))) break;
                    tc_fence_after();
                    const uint32_t tX = tmem + 128u * (uint32_t)half + lane_off;
#pragma unroll 1
                    for (int c8 = 0; c8 < 2; ++c8) {
                        const int ql0 = 32 * c8, i0 = q0 + 64 * half + ql0;  // queries i0 .. i0+31
                        const bool live = jmin < L.S && i0 < L.S && i0 + 31 >= jmin && i0 <= jmax + L.W - 1;
                        const bool full = jmax <= i0 && jmin > i0 + 31 - L.W && i0 + 31 < L.S && jmax < L.S;
                        uint32_t pp[16], dd[16];
                        if (live) {
                            float sv[32], dv[32];
                            tmem_ld32f(tX + 32 * c8, sv);
                            tmem_ld32f(tX + 64 + 32 * c8, dv);
                            tmem_wait_ld();
                            if (full) {
                                kv_chunk<true>(sv, dv, sm.lsec[slot] + ql0, sm.delta[slot] + ql0, sm.dcol[slot] + ql0, 0u,
                                               vin, su, dsc, c2, pp, dd, kacc);
                            } else {
                                // queries that see key j: j <= i <= min(j + W - 1, S - 1)
                                const uint32_t vm = j < L.S ? bit_range(j - i0, min(j + L.W - 1, L.S - 1) - i0) : 0u;
                                kv_chunk<false>(sv, dv, sm.lsec[slot] + ql0, sm.delta[slot] + ql0, sm.dcol[slot] + ql0, vm,
                                                vin, su, dsc, c2, pp, dd, kacc);
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) pp[e] = dd[e] = 0u;
                        }
                        tmem_st16(tX + 16 * c8, pp);       // P^T over S^T (already read)
                        tmem_st16(tX + 64 + 16 * c8, dd);  // dS^T over dP^T
                    }
                    if (it == x.nit - 1) sm.kmdot[my_half][uu & 1][r] = kacc * mdot_f;  // the epilogue adds both
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&sm.bar[KB_PFULL + half]);
                }
            }
        }
    } else if (warp >= 12) {
        reg_alloc<192>();
        // ================================================ unit scales; dv, dk epilogue (thread = key row)
        const int r = tid - 384, wq = warp - 12;
        const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
        int uu = 0;
        // Scales of unit x into ring slot `slot`: max |dout| and max |Delta| over the rows the
        // unit reads (global loads only), the dA scale E, the dS^T row scales and the V tile
        // scale.  This warpgroup is otherwise idle during a unit: it computes the next unit's
        // scales right after the previous unit's epilogue, and hands them to the softmax
        // through KB_STATS (two barriers alternating by unit, so neither runs a phase ahead).
        int n_red = 0;
        auto unit_scales = [&](const UnitInfo& x, int slot) -> bool {
            // every global load of the unit's statistics is issued before any is used (one
            // round trip instead of one per dependent batch)
            const int j = x.kt * TF_BN + r, nkt = (L.S + TF_BN - 1) / TF_BN;
            const float vnorm = j < L.S ? p.vnorm[((size_t)x.b * L.Hkv + x.kvh) * L.S + j] : 0.f;
            const float vtile = p.vtinv[((size_t)x.b * L.Hkv + x.kvh) * nkt + x.kt];
            float domx = 0.f, dlmx = 0.f;
            if constexpr (WIDE) {
                // per-tile maxima over the query blocks qb0 .. qb0 + nit/G - 1 (bwd_tile_stats_kernel)
                const size_t nst = (size_t)L.B * L.Hkv * nkt, base = ((size_t)x.b * L.Hkv + x.kvh) * nkt;
                for (int t = x.qb0 + r; t < x.qb0 + x.nit / L.G; t += TF_BN) {
                    domx = fmaxf(domx, p.tstat[base + t]);
                    dlmx = fmaxf(dlmx, p.tstat[nst + base + t]);
                }
            }
            for (int it0 = 0; !WIDE && it0 < x.nit; it0 += 8) {
                float dm[8], dl[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    dm[k] = 0.f;
                    dl[k] = 0.f;
                    int qb, hg;
                    decode_iter(L, x, it0 + k, qb, hg);
                    const int i = qb * TF_BM + r;
                    if (it0 + k < x.nit && i < L.S) {
                        const size_t rp = ((size_t)x.b * L.Hq + hg) * row_stride(L.S) + i;
                        dm[k] = p.domax[rp];
                        dl[k] = p.P.delta[rp];
                    }
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    domx = fmaxf(domx, dm[k]);
                    dlmx = fmaxf(dlmx, fabsf(dl[k]));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                domx = fmaxf(domx, __shfl_xor_sync(0xffffffffu, domx, o));
                dlmx = fmaxf(dlmx, __shfl_xor_sync(0xffffffffu, dlmx, o));
            }
            // across the 4 warps through an mbarrier (a bounded wait: a named barrier would hang
            // if some thread had given up earlier); the scratch alternates by call parity
            float(*rr)[4] = sm.red[n_red & 1];
            if (lane == 0) {
                rr[0][wq] = domx;
                rr[1][wq] = dlmx;
                mbar_arrive(&sm.bar[KB_RED]);
            }
            if (!mbar_wait(&sm.bar[KB_RED], n_red & 1, abort, 232)) return false;
            ++n_red;
            domx = fmaxf(fmaxf(rr[0][0], rr[0][1]), fmaxf(rr[0][2], rr[0][3]));
            dlmx = fmaxf(fmaxf(rr[1][0], rr[1][1]), fmaxf(rr[1][2], rr[1][3]));
            // E = fit_exp(max domax) is the smallest row exponent of dA in the unit, so every
            // column factor 2^(E - e_i) of P^T is <= 1
            const int E = fit_exp(domx);
            // dS^T row scale: |dS_ji| <= |v_j| |dA_i| + |Delta_i| <= |v_j| sqrt(D) max|dout| + max|Delta|
            sm.dsc[slot][r] = ldexpf(1.0f, fit_exp(vnorm * sqrtf((float)kD) * domx + dlmx));
            if (r == 0) {
                sm.uinv[slot] = ldexpf(1.0f, -E);
                sm.vtinv[slot] = vtile;
            }
            return true;
        };
        bool ok = true;
        if (u_begin < u_end && (ok = unit_scales(decode_unit(L, u_begin, WIDE), 0))) mbar_arrive(&sm.bar[KB_STATS]);
        for (int u = u_begin; u < u_end && ok; ++u, ++uu) {
            if (u + 1 < u_end) {
                if (!(ok = unit_scales(decode_unit(L, u + 1, WIDE), (uu + 1) & 3))) break;
                mbar_arrive(&sm.bar[KB_STATS + ((uu + 1) & 1)]);
            }
            const UnitInfo x = decode_unit(L, u, WIDE);
            const int j = x.kt * TF_BN + r;
            const bool valid = j < L.S;
            const size_t off = ((size_t)(x.b * (size_t)L.S + (valid ? j : 0)) * L.Hkv + x.kvh) * kD;
            uint4 xv0[8];  // first half of the raw k row, in flight during the wait
#pragma unroll
            for (int c = 0; c < 8; ++c)
                xv0[c] = valid ? __ldg(reinterpret_cast<const uint4*>(L.k + off) + c) : make_uint4(0u, 0u, 0u, 0u);
            if (!mbar_wait(&sm.bar[KB_DVKFULL], uu & 1, abort, 240)) break;
            tc_fence_after();
            const float dvf = sm.uinv[uu & 3];
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float v[32];
                tmem_ld32f(TM_DV + lane_off + 32 * c, v);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) o[e] = pack_bf16(v[8 * q4 + 2 * e] * dvf, v[8 * q4 + 2 * e + 1] * dvf);
                        reinterpret_cast<uint4*>(p.P.dv + off)[4 * c + q4] = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
            float dy[128];
            tmem_ld32f(TM_DK + lane_off, dy);
            tmem_ld32f(TM_DK + lane_off + 32, dy + 32);
            tmem_ld32f(TM_DK + lane_off + 64, dy + 64);
            tmem_ld32f(TM_DK + lane_off + 96, dy + 96);
            tmem_wait_ld();
            const float f = L.scale / (sm.dsc[uu & 3][r] * oscale);
            const float mdot = sm.kmdot[0][uu & 1][r] + sm.kmdot[1][uu & 1][r];
            const float rinv = valid ? p.krinv[((size_t)x.b * L.Hkv + x.kvh) * L.S + j] : 0.f;
            tc_fence_before();
            mbar_arrive(&sm.bar[KB_DVKEMPTY]);  // dV, dK of the unit are out of TMEM
            row_rope_rms_backward_regs<ANY ? 0 : TF_HALF>(dy, f, mdot, rinv, xv0, L.k + off, p.P.dk + off, valid, j,
                                                          sm.gk, sm.dgk[wq], L);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
    if (tid < kD)
        p.P.dgk_part[(size_t)blockIdx.x * kD + tid] = (sm.dgk[0][tid] + sm.dgk[1][tid]) + (sm.dgk[2][tid] + sm.dgk[3][tid]);
    if (tid == 0 && sm.abort && p.err) atomicExch(p.err, sm.abort);
}

// =====================================================================  host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_b() {
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

bool make_map_b(CUtensorMap* map, const void* base, int H, int S, int B,
                CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, int box_rows = 128) {
    auto enc = get_encode_b();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)S * H * kD * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 map {Spad, H, B} of a padded per-row array, box {64, 1, 1}, no swizzle
bool make_map_rows(CUtensorMap* map, const float* base, int H, int Spad, int B) {
    auto enc = get_encode_b();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)Spad, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)Spad * 4, (cuuint64_t)H * Spad * 4};
    cuuint32_t box[3] = {64, 1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern const char* const kBwdTcKernelNames[] = {"bwd_gate_kernel",         "bwd_prep_kv_kernel",
                                                "bwd_prep_q_kernel",       "bwd_q_tc_kernel",
                                                "bwd_kv_tc_kernel",        "dgamma_reduce_kernel(k)",
                                                "dgamma_reduce_kernel(q)"};
extern const int kBwdTcKernelCount = 7;
extern const char* const kBwdWideKernelNames[] = {"bwd_gate_kernel",       "bwd_prep_kv_kernel",
                                                  "bwd_prep_q_kernel",     "bwd_tile_stats_kernel",
                                                  "bwd_q_glob_kernel",     "bwd_kv_tc_kernel",
                                                  "dgamma_reduce_kernel(k)", "dgamma_reduce_kernel(q)"};
extern const int kBwdWideKernelCount = 8;
// the same given the forward's saved Q~, K~ and inverse RMS: V alone is prepared
extern const char* const kBwdTcSavedKernelNames[] = {"bwd_gate_kernel",  "bwd_prep_v_kernel",
                                                     "bwd_q_tc_kernel",  "bwd_kv_tc_kernel",
                                                     "dgamma_reduce_kernel(k)", "dgamma_reduce_kernel(q)"};
extern const int kBwdTcSavedKernelCount = 6;
extern const char* const kBwdWideSavedKernelNames[] = {"bwd_gate_kernel",   "bwd_prep_v_kernel",
                                                       "bwd_tile_stats_kernel", "bwd_q_glob_kernel",
                                                       "bwd_kv_tc_kernel",  "dgamma_reduce_kernel(k)",
                                                       "dgamma_reduce_kernel(q)"};
extern const int kBwdWideSavedKernelCount = 7;

// d_gamma[d] = sum over the n partial rows parts[i][d] (one per CTA of the kernel that wrote
// them), in a fixed order so repeated runs give the same bits: eight groups of 128 threads
// take every eighth row, then group 0 adds the eight group sums.  One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) dgamma_reduce_kernel(const float* __restrict__ parts, int n,
                                                             float* __restrict__ out) {
    __shared__ float acc[8][kD];
    const int d = threadIdx.x & (kD - 1), grp = threadIdx.x >> 7;
    float s = 0.f;
    for (int i = grp; i < n; i += 8) s += parts[(size_t)i * kD + d];
    acc[grp][d] = s;
    __syncthreads();
    if (grp == 0) {
        float t = 0.f;
#pragma unroll
        for (int g2 = 0; g2 < 8; ++g2) t += acc[g2][d];
        out[d] = t;
    }
}

// Windows up to one key tile, any rotated dims and group size.  A shape test only: without
// the driver's tensor-map encoder the launch fails (ZGCM_ERR_CUDA).
bool bwd_tc_supported(const LayerParams& L) {
    return L.W <= TF_BN && L.S >= 1 && L.B >= 1;
}

// Windows wider than one tile (the global layer among them), any rotated dims.  A shape test
// only: without the driver's tensor-map encoder the launch fails (ZGCM_ERR_CUDA).
bool bwd_wide_supported(const LayerParams& L) {
    return L.W > TF_BN && L.S >= 1 && L.B >= 1;
}

namespace {
// d_gamma partial-sum slots: the persistent sliding-window kernels use at most TB_MAX_GRID
// CTAs, the wide-window ones one CTA per unit (at most B*Hq*ceil(S/128))
size_t dgamma_slots(int B, int S, int Hq) {
    const size_t units = (size_t)B * Hq * ((S + TF_BM - 1) / TF_BM);
    return units > (size_t)TB_MAX_GRID ? units : (size_t)TB_MAX_GRID;
}
}  // namespace

// workspace of the tcgen05 backward: delta, domax, dainv, lse2p [B,Hq,Spad] and qrinv
// [B,Hq,S] fp32; dA16, Q~16
// [B,S,Hq,D] fp16; K~16, V16 [B,S,Hkv,D] fp16; krinv, vnorm [B,Hkv,S] fp32; vtinv per V
// tile; per-tile maxima (wide windows); 2 x d_gamma partials
size_t bwd_tc_workspace_bytes(int B, int S, int Hq, int Hkv) {
    const size_t rows = (size_t)B * S * Hq, krows = (size_t)B * S * Hkv;
    const size_t prows = (size_t)B * Hq * row_stride(S);  // padded row arrays
    const size_t tiles = (size_t)B * Hkv * ((S + TF_BN - 1) / TF_BN);
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    return 4 * a(prows * sizeof(float)) + a(rows * sizeof(float)) + 2 * a(rows * kD * sizeof(__half)) +
           2 * a(krows * kD * sizeof(__half)) + 2 * a(krows * sizeof(float)) + a(tiles * sizeof(float)) +
           a(3 * tiles * sizeof(float)) + 2 * a(dgamma_slots(B, S, Hq) * kD * sizeof(float));
}

// Q~ fp16 [B,S,Hq,D] into q16 and each q row's inverse RMS into qrinv ([B,Hq,S]): the
// backward's query preparation, run by a forward that keeps its activations.
cudaError_t launch_prep_q_only(const LayerParams& L, void* q16, float* qrinv, int* err_word, cudaStream_t stream) {
    BwdTcParams p;
    p.P.L = L;
    p.qrinv = qrinv;
    p.err = err_word;
    const long long q_tiles = (long long)L.B * L.Hq * ((L.S + TF_BN - 1) / TF_BN);
    if (q_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (!make_map_b(&p.tm_q, L.q, L.Hq, L.S, L.B) ||
        !make_map_b(&p.tm_q16, q16, L.Hq, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return cudaErrorInvalidValue;
    const size_t smem_pq = sizeof(PrepSmem<false>) + 1024;
    auto prep_q = L.rope_half != TF_HALF ? bwd_prep_q_kernel<true> : bwd_prep_q_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(prep_q, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_pq);
    if (e != cudaSuccess) return e;
    prep_q<<<(int)q_tiles, KP_THREADS, smem_pq, stream>>>(p);
    return cudaGetLastError();
}

// With `sv`, Q~, K~ and the rows' inverse RMS come from the forward: the K/V preparation
// converts V alone and the Q preparation does not run.
cudaError_t launch_bwd_tc(const BwdParams& bp, void* workspace, int* err_word, cudaStream_t stream,
                          void* const* events, int n_pairs, const SavedAct* sv) {
    BwdTcParams p;
    p.P = bp;
    // a window of S or more is the full causal one: clamped so that window arithmetic
    // (j + W - 1) stays in range
    if (p.P.L.W > p.P.L.S) p.P.L.W = p.P.L.S;
    const LayerParams& L = p.P.L;
    const size_t rows = (size_t)L.B * L.S * L.Hq;
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    char* ws = static_cast<char*>(workspace);
    size_t off = 0;
    auto take = [&](size_t bytes) -> char* {
        char* q = ws + off;
        off += a(bytes);
        return q;
    };
    const int Spad = row_stride(L.S);
    const size_t prows = (size_t)L.B * L.Hq * Spad;
    p.P.delta = reinterpret_cast<float*>(take(prows * 4));
    p.domax = reinterpret_cast<float*>(take(prows * 4));
    p.dainv = reinterpret_cast<float*>(take(prows * 4));
    p.lse2p = reinterpret_cast<float*>(take(prows * 4));
    __half* da16 = reinterpret_cast<__half*>(take(rows * kD * sizeof(__half)));
    p.da16 = da16;
    void* q16 = take(rows * kD * sizeof(__half));
    p.qrinv = reinterpret_cast<float*>(take(rows * 4));
    const size_t krows = (size_t)L.B * L.S * L.Hkv;
    const int nkt = (L.S + TF_BN - 1) / TF_BN;
    void* k16 = take(krows * kD * sizeof(__half));
    void* v16 = take(krows * kD * sizeof(__half));
    p.krinv = reinterpret_cast<float*>(take(krows * 4));
    p.vnorm = reinterpret_cast<float*>(take(krows * 4));
    p.vtinv = reinterpret_cast<float*>(take((size_t)L.B * L.Hkv * nkt * 4));
    p.tstat = reinterpret_cast<float*>(take(3 * (size_t)L.B * L.Hkv * nkt * 4));
    const size_t slots = dgamma_slots(L.B, L.S, L.Hq);
    p.P.dgq_part = reinterpret_cast<float*>(take(slots * kD * 4));
    p.P.dgk_part = reinterpret_cast<float*>(take(slots * kD * 4));
    if (sv) {
        q16 = sv->q16;
        p.qrinv = sv->qrinv;
        k16 = sv->k16;
        p.krinv = sv->krinv;
    }
    p.err = err_word;
    const bool wide = bp.L.W > TF_BN;  // as the kernel-name query decides: on the window given
    p.wide = wide ? 1 : 0;
    if (!make_map_b(&p.tm_q, L.q, L.Hq, L.Sq, L.B) || !make_map_b(&p.tm_k, L.k, L.Hkv, L.S, L.B) ||
        !make_map_b(&p.tm_v, L.v, L.Hkv, L.S, L.B) ||
        !make_map_b(&p.tm_da, da16, L.Hq, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_map_b(&p.tm_k16, k16, L.Hkv, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_map_b(&p.tm_v16, v16, L.Hkv, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_map_b(&p.tm_q16, q16, L.Hq, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_map_b(&p.tm_q16h, q16, L.Hq, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 64) ||
        !make_map_b(&p.tm_dah, da16, L.Hq, L.S, L.B, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 64) ||
        !make_map_rows(&p.tm_lse, p.lse2p, L.Hq, Spad, L.B) || !make_map_rows(&p.tm_delta, p.P.delta, L.Hq, Spad, L.B) ||
        !make_map_rows(&p.tm_dainv, p.dainv, L.Hq, Spad, L.B))
        return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    sms = sms < TB_MAX_GRID ? sms : TB_MAX_GRID;
    const size_t smem_q = sizeof(BwdQTcSmem) + 1024, smem_k = sizeof(BwdKTcSmem) + 1024;
    // the layer's 21 rotated pairs take the unrolled instances, any other number the general ones
    const bool any = L.rope_half != TF_HALF;
    auto q_tc = any ? bwd_q_tc_kernel<true> : bwd_q_tc_kernel<false>;
    auto kv_slide = any ? bwd_kv_tc_kernel<false, true> : bwd_kv_tc_kernel<false, false>;
    auto kv_wide = any ? bwd_kv_tc_kernel<true, true> : bwd_kv_tc_kernel<true, false>;
    auto prep_kv = any ? bwd_prep_kv_kernel<true> : bwd_prep_kv_kernel<false>;
    auto prep_q = any ? bwd_prep_q_kernel<true> : bwd_prep_q_kernel<false>;
    if ((e = cudaFuncSetAttribute(q_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_q)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(kv_slide, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_k)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(kv_wide, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_k)) != cudaSuccess)
        return e;
    // events[2i] / events[2i+1] bracket kernel i (i < n_pairs)
    auto before = [&](int i) -> cudaError_t {
        return i < n_pairs ? cudaEventRecord(static_cast<cudaEvent_t>(events[2 * i]), stream) : cudaSuccess;
    };
    auto after = [&](int i) -> cudaError_t {
        cudaError_t le = cudaGetLastError();
        if (le != cudaSuccess) return le;
        return i < n_pairs ? cudaEventRecord(static_cast<cudaEvent_t>(events[2 * i + 1]), stream) : cudaSuccess;
    };
    const int nqb = (L.S + TF_BM - 1) / TF_BM;
    const long long steps = (long long)L.B * L.Hkv * nqb;  // query-major steps = key-major units
    if (steps > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.total = (int)steps;
    const int grid = (int)(steps < sms ? steps : sms);
    // gate pass over the query rows: 4 resident blocks of 256 threads per SM, each half-warp
    // GATE_UNROLL rows at a time
    const long long qrows = (long long)L.B * L.Sq * L.Hq;
    const long long half_warps = (qrows + GATE_UNROLL - 1) / GATE_UNROLL;
    const long long gate_need = (half_warps * 16 + GATE_THREADS - 1) / GATE_THREADS;
    const int gate_grid = (int)(gate_need < 4LL * sms ? gate_need : 4LL * sms);
    const size_t smem_pk = sizeof(PrepSmem<true>) + 1024, smem_pq = sizeof(PrepSmem<false>) + 1024;
    if ((e = cudaFuncSetAttribute(prep_kv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_pk)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(prep_q, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_pq)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(bwd_prep_v_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_pk)) !=
        cudaSuccess)
        return e;
    const long long k_tiles = (long long)L.B * L.Hkv * nkt;
    const long long q_tiles = (long long)L.B * L.Hq * ((L.Sq + TF_BN - 1) / TF_BN);  // of the query rows
    if (q_tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    int i = 0;
    if ((e = before(i)) != cudaSuccess) return e;
    if (wide)
        bwd_gate_kernel<true><<<gate_grid, GATE_THREADS, 0, stream>>>(bp.dout, L.g, bp.out, bp.dg, da16, p.dainv,
                                                                      p.domax, p.P.delta, qrows, L.S, L.Hq, L.q_off);
    else
        bwd_gate_kernel<false><<<gate_grid, GATE_THREADS, 0, stream>>>(bp.dout, L.g, bp.out, bp.dg, da16, p.dainv,
                                                                       p.domax, nullptr, qrows, L.S, L.Hq, 0);
    if ((e = after(i++)) != cudaSuccess) return e;
    if ((e = before(i)) != cudaSuccess) return e;
    if (sv)
        bwd_prep_v_kernel<<<(int)k_tiles, KP_THREADS, smem_pk, stream>>>(p);
    else
        prep_kv<<<(int)k_tiles, KP_THREADS, smem_pk, stream>>>(p);
    if ((e = after(i++)) != cudaSuccess) return e;
    if (!sv) {
        if ((e = before(i)) != cudaSuccess) return e;
        prep_q<<<(int)q_tiles, KP_THREADS, smem_pq, stream>>>(p);
        if ((e = after(i++)) != cudaSuccess) return e;
    }
    if (wide) {
        // per-tile bounds, then the query-major sweep (one CTA per (b, head, block), heaviest
        // first) and the key-major one (one CTA per (b, KV head, tile), heaviest first)
        // query blocks from the one of the first query row on; key tiles from the first one
        // a query row sees (wide_first_tile), the ones before it get zero dk and dv
        const long long units_q = (long long)L.B * L.Hq * (nqb - L.q_off / TF_BM);
        const int kt0 = wide_first_tile(L);
        const long long units_k = (long long)L.B * L.Hkv * (nkt - kt0);
        if (kt0 > 0) {
            const size_t pitch = (size_t)L.S * L.Hkv * kD * sizeof(bf16);
            const size_t width = (size_t)kt0 * TF_BN * L.Hkv * kD * sizeof(bf16);
            if ((e = cudaMemset2DAsync(bp.dk, pitch, 0, width, L.B, stream)) != cudaSuccess) return e;
            if ((e = cudaMemset2DAsync(bp.dv, pitch, 0, width, L.B, stream)) != cudaSuccess) return e;
        }
        if ((e = before(i)) != cudaSuccess) return e;
        bwd_tile_stats_kernel<<<(int)k_tiles, BTS_THREADS, 0, stream>>>(p);
        if ((e = after(i++)) != cudaSuccess) return e;
        if ((e = before(i)) != cudaSuccess) return e;
        if ((e = launch_bwd_q_glob(p, (int)units_q, stream)) != cudaSuccess) return e;
        if ((e = after(i++)) != cudaSuccess) return e;
        p.total = (int)units_k;
        if ((e = before(i)) != cudaSuccess) return e;
        kv_wide<<<(int)units_k, TB_THREADS, smem_k, stream>>>(p);
        if ((e = after(i++)) != cudaSuccess) return e;
        if ((e = before(i)) != cudaSuccess) return e;
        dgamma_reduce_kernel<<<1, 1024, 0, stream>>>(p.P.dgk_part, (int)units_k, bp.dgamma_k);
        if ((e = after(i++)) != cudaSuccess) return e;
        if ((e = before(i)) != cudaSuccess) return e;
        dgamma_reduce_kernel<<<1, 1024, 0, stream>>>(p.P.dgq_part, (int)units_q, bp.dgamma_q);
        return after(i);
    }
    if ((e = before(i)) != cudaSuccess) return e;
    q_tc<<<grid, TB_THREADS, smem_q, stream>>>(p);
    if ((e = after(i++)) != cudaSuccess) return e;
    if ((e = before(i)) != cudaSuccess) return e;
    kv_slide<<<grid, TB_THREADS, smem_k, stream>>>(p);
    if ((e = after(i++)) != cudaSuccess) return e;
    if ((e = before(i)) != cudaSuccess) return e;
    dgamma_reduce_kernel<<<1, 1024, 0, stream>>>(p.P.dgk_part, grid, bp.dgamma_k);
    if ((e = after(i++)) != cudaSuccess) return e;
    if ((e = before(i)) != cudaSuccess) return e;
    dgamma_reduce_kernel<<<1, 1024, 0, stream>>>(p.P.dgq_part, grid, bp.dgamma_q);
    return after(i);
}

}  // namespace zgcm
