// bwd_mma.cu — gated window-attention backward on the warp-level tensor-core path
// (mma.sync m16n8k16 bf16 -> fp32).  Exact gradients of L = sum(dout * out) for the
// ZGCM-1 layer (definition and page citations in common.cuh).
//
// Kernels, in launch order:
//   bwd_pre     per (b, s, h) row: dg = dout*out*(1-sigmoid(g)); dA = dout*sigmoid(g)
//               (out = sigmoid(g)*A, so neither needs the pre-gate A itself).
//   bwd_dq      per (b, query head, 64-query tile), two passes over the key tiles its
//               window reaches.  Pass 1: the tile's own log-sum-exp (online max and sum)
//               and Delta = sum_j P dP with P = exp(S - lse), dP = dA V^T.  Pass 2:
//               dS = P (dP - Delta), dQ~ = scale dS K~.  Epilogue: dq = RMSNorm/RoPE
//               backward of dQ~, d_gamma_q partials; lse and Delta saved for bwd_main.
//   bwd_main    per (b, KV head, 64-key tile), over the Hq/Hkv query heads of the group and
//               every 64-query tile whose window reaches the keys:
//                 P^T = exp(S^T - lse), dV += P^T dA, dP^T = V dA^T, dS^T = P^T (dP^T - Delta),
//                 dK~ += dS^T Q~;  epilogue: dk = RMSNorm/RoPE backward of scale dK~, dv,
//                 d_gamma_k partials.
//   dgamma      fixed-order sum of the partials (deterministic).
//
// Precision.  The stated bound is max-abs 2e-2 on bf16 gradients whose largest entries
// (|x| ~ 4..6, where one bf16 rounding alone costs up to 0.0156) sit at the start of a
// sequence, where a handful of keys share the softmax and a few products dominate each
// sum.  Measured against the fp64 oracle in a CPU emulation of these kernels, three things
// were needed to stay inside it:
//   * Delta is formed from the kernels' own P and dP, and lse from their own scores (not
//     from dout*out with a bf16 `out`, nor from the forward's lse): otherwise P and Delta
//     are inconsistent with dP and the worst dk error doubles;
//   * dS in the direct form P (dP - Delta): the one-pass sum_j P dP k~ - Delta sum_j P k~
//     cancels where the softmax is peaked (one-key windows, the first tokens);
//   * every operand of a gradient product is carried as a bf16 pair hi + lo
//     (hi = bf16(x), lo = bf16(x - hi)) and the product as hi*hi + hi*lo + lo*hi:
//     dA in dP and dV, P in dV, dS and q~ in dK, dS and k~ in dQ.
// The scores S = q~ k~^T use the bf16 q~, k~ (hi) in both kernels, as the forward does.
#include "common.cuh"

namespace zgcm {

// =====================================================================  bwd_pre

constexpr int PRE_WARPS = 8;

__global__ void __launch_bounds__(PRE_WARPS * 32) bwd_pre_kernel(const __grid_constant__ BwdParams p) {
    const LayerParams& L = p.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long nrows = (long long)L.B * L.S * L.Hq;
    const long long row = (long long)blockIdx.x * PRE_WARPS + warp;
    if (row >= nrows) return;
    const size_t off = (size_t)row * kD + 4 * lane;
    uint2 dor = *reinterpret_cast<const uint2*>(p.dout + off);
    uint2 outr = *reinterpret_cast<const uint2*>(p.out + off);
    uint2 gr = *reinterpret_cast<const uint2*>(L.g + off);
    float d[4], o[4], g[4];
    {
        float2 a = unpack_bf16(dor.x), b = unpack_bf16(dor.y);
        d[0] = a.x; d[1] = a.y; d[2] = b.x; d[3] = b.y;
        a = unpack_bf16(outr.x); b = unpack_bf16(outr.y);
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
        a = unpack_bf16(gr.x); b = unpack_bf16(gr.y);
        g[0] = a.x; g[1] = a.y; g[2] = b.x; g[3] = b.y;
    }
    float dgv[4], dav[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float sg = sigmoidf_(g[e]);
        dgv[e] = d[e] * o[e] * (1.f - sg);
        dav[e] = d[e] * sg;
    }
    *reinterpret_cast<uint2*>(p.dg + off) = make_uint2(pack_bf16(dgv[0], dgv[1]), pack_bf16(dgv[2], dgv[3]));
    const uint32_t h01 = pack_bf16(dav[0], dav[1]), h23 = pack_bf16(dav[2], dav[3]);
    const float2 r01 = unpack_bf16(h01), r23 = unpack_bf16(h23);
    *reinterpret_cast<uint2*>(p.dA + off) = make_uint2(h01, h23);
    *reinterpret_cast<uint2*>(p.dA_lo + off) =
        make_uint2(pack_bf16(dav[0] - r01.x, dav[1] - r01.y), pack_bf16(dav[2] - r23.x, dav[3] - r23.y));
}

// =====================================================================  shared helpers

// store this lane's 4 values of `row` as bf16 hi (and lo = bf16(y - hi) when lo != null)
__device__ __forceinline__ void store_row_split(bf16* hi, bf16* lo, int row, const float y[4]) {
    const int lane = threadIdx.x & 31;
    const uint32_t off = tile_off(row, lane >> 1) + (lane & 1) * 8;
    const uint32_t h01 = pack_bf16(y[0], y[1]), h23 = pack_bf16(y[2], y[3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<char*>(hi) + off) = make_uint2(h01, h23);
    if (lo) {
        const float2 a = unpack_bf16(h01), b = unpack_bf16(h23);
        *reinterpret_cast<uint2*>(reinterpret_cast<char*>(lo) + off) =
            make_uint2(pack_bf16(y[0] - a.x, y[1] - a.y), pack_bf16(y[2] - b.x, y[3] - b.y));
    }
}

// A-fragments (hi, lo) of a 16x16 slice of fp32 accumulators c[2 kk], c[2 kk + 1]
__device__ __forceinline__ void split_frag(const float (*c)[4], int kk, uint32_t hi[4], uint32_t lo[4]) {
    const float* f[4] = {&c[2 * kk][0], &c[2 * kk][2], &c[2 * kk + 1][0], &c[2 * kk + 1][2]};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        hi[u] = pack_bf16(f[u][0], f[u][1]);
        const float2 h = unpack_bf16(hi[u]);
        lo[u] = pack_bf16(f[u][0] - h.x, f[u][1] - h.y);
    }
}

// =====================================================================  bwd_dq

constexpr int DQ_BM = 64;       // query rows per CTA (4 warps x 16)
constexpr int DQ_BN = 64;       // keys per tile
constexpr int DQ_THREADS = 128;

struct BwdDqSmem {
    bf16 Q[DQ_BM * kD];         // Q~ (normalised + rotated), swizzled rows
    bf16 dA[DQ_BM * kD];
    bf16 dAl[DQ_BM * kD];
    bf16 K[2][DQ_BN * kD];      // K~ hi
    bf16 Kl[2][DQ_BN * kD];     // K~ lo
    bf16 V[2][DQ_BN * kD];
    float ybuf[DQ_THREADS / 32][kD];
    float gq[kD], gk[kD];
    float dgq[DQ_THREADS / 32][kD];
};
static_assert(DQ_BM * kD * 4 <= sizeof(bf16) * 2 * DQ_BN * kD, "dQ staging fits in the K buffers");

// K~ (hi, lo) prologue (16 rows per warp) + V via cp.async for the key tile at kbase.
__device__ __forceinline__ void dq_load_kv(const LayerParams& L, BwdDqSmem& sm, int buf, int b, int kvh,
                                           int kbase) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int c = tid + DQ_THREADS * i;
        int row = c >> 4, ch = c & 15, pos = kbase + row;
        bool ok = pos < L.S;
        const bf16* src = L.v + ((size_t)(b * (size_t)L.S + (ok ? pos : 0)) * L.Hkv + kvh) * kD + ch * 8;
        cp_async16(smem_u32(reinterpret_cast<char*>(sm.V[buf]) + tile_off(row, ch)), src, ok);
    }
    cp_async_commit();
    uint2 raw[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        int pos = kbase + warp * 16 + r;
        raw[r] = pos < L.S ? load_row4(L.k + ((size_t)(b * (size_t)L.S + pos) * L.Hkv + kvh) * kD)
                           : make_uint2(0u, 0u);
    }
    const float g4[4] = {sm.gk[4 * lane], sm.gk[4 * lane + 1], sm.gk[4 * lane + 2], sm.gk[4 * lane + 3]};
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        int row = warp * 16 + r, pos = kbase + row;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
        if (pos < L.S) prologue_row(raw[r], g4, L, pos, sm.ybuf[warp], y);
        store_row_split(sm.K[buf], sm.Kl[buf], row, y);
    }
}

__global__ void __launch_bounds__(DQ_THREADS, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
    const LayerParams& L = p.L;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    BwdDqSmem& sm = *reinterpret_cast<BwdDqSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int nqt = (L.S + DQ_BM - 1) / DQ_BM;
    int bid = blockIdx.x;
    const int b = bid / (nqt * L.Hq);
    bid -= b * nqt * L.Hq;
    const int h = bid / nqt;
    int qt = bid - h * nqt;
    if (L.W >= L.S) qt = nqt - 1 - qt;  // full causal: longest rows first
    const int kvh = h / L.G;
    const int q0 = qt * DQ_BM;

    if (tid < kD) {
        sm.gq[tid] = L.gamma_q[tid];
        sm.gk[tid] = L.gamma_k[tid];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int c = tid + DQ_THREADS * i;
        int row = c >> 4, ch = c & 15, pos = q0 + row;
        bool ok = pos < L.S;
        const size_t go = ((size_t)(b * (size_t)L.S + (ok ? pos : 0)) * L.Hq + h) * kD + ch * 8;
        cp_async16(smem_u32(reinterpret_cast<char*>(sm.dA) + tile_off(row, ch)), p.dA + go, ok);
        cp_async16(smem_u32(reinterpret_cast<char*>(sm.dAl) + tile_off(row, ch)), p.dA_lo + go, ok);
    }
    cp_async_commit();
    __syncthreads();
    const float gq4[4] = {sm.gq[4 * lane], sm.gq[4 * lane + 1], sm.gq[4 * lane + 2], sm.gq[4 * lane + 3]};
    {
        uint2 raw[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            int pos = q0 + warp * 16 + r;
            raw[r] = pos < L.S ? load_row4(L.q + ((size_t)(b * (size_t)L.S + pos) * L.Hq + h) * kD)
                               : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            int row = warp * 16 + r, pos = q0 + row;
            float y[4] = {0.f, 0.f, 0.f, 0.f};
            if (pos < L.S) prologue_row(raw[r], gq4, L, pos, sm.ybuf[warp], y);
            store_row_split(sm.Q, nullptr, row, y);
        }
    }

    const int klo = max(0, q0 - L.W + 1);
    const int khi = min(L.S - 1, q0 + DQ_BM - 1);
    const int kt_lo = klo / DQ_BN, kt_hi = khi / DQ_BN;
    const int wq0 = q0 + warp * 16;
    const int r0 = wq0 + (lane >> 2), r1 = r0 + 8;

    float dq[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[i][e] = 0.f;
    // pass-1 statistics of rows r0, r1 (base-2 scores): running max, and this thread's
    // partial sums of exp2(s - max) and of exp2(s - max) * dP
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f, n0 = 0.f, n1 = 0.f;
    float lse0 = INFINITY, lse1 = INFINITY, del0 = 0.f, del1 = 0.f;
    const int ntiles = kt_hi - kt_lo + 1;

    dq_load_kv(L, sm, 0, b, kvh, kt_lo * DQ_BN);
    for (int it = 0; it < 2 * ntiles; ++it) {
        const int pass = it >= ntiles ? 1 : 0;
        const int kt = kt_lo + (it - pass * ntiles);
        const int buf = it & 1;
        cp_async_wait<0>();
        __syncthreads();
        if (it + 1 < 2 * ntiles) dq_load_kv(L, sm, buf ^ 1, b, kvh, (kt_lo + ((it + 1) % ntiles)) * DQ_BN);
        if (it == ntiles) {
            // pass 1 complete: row sums over the quad of lanes holding each row
            l0 += __shfl_xor_sync(0xffffffffu, l0, 1); l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 1); l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
            n0 += __shfl_xor_sync(0xffffffffu, n0, 1); n0 += __shfl_xor_sync(0xffffffffu, n0, 2);
            n1 += __shfl_xor_sync(0xffffffffu, n1, 1); n1 += __shfl_xor_sync(0xffffffffu, n1, 2);
            if (l0 > 0.f) { lse0 = m0 + log2f(l0); del0 = n0 / l0; }
            if (l1 > 0.f) { lse1 = m1 + log2f(l1); del1 = n1 / l1; }
        }
        const int kbase = kt * DQ_BN;
        const bool live = wq0 < L.S && kbase <= wq0 + 15 && kbase + DQ_BN - 1 >= wq0 - L.W + 1;
        if (!live) continue;
        const uint32_t qs = smem_u32(sm.Q), das = smem_u32(sm.dA), dls = smem_u32(sm.dAl),
                       ks = smem_u32(sm.K[buf]), kls = smem_u32(sm.Kl[buf]), vs = smem_u32(sm.V[buf]);
        float s[8][4], dp[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
        // S = Q~ K~^T and dP = (dA_hi + dA_lo) V^T  (16 queries x 64 keys per warp)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t aq[4], ad[4], al[4];
            const uint32_t ao = tile_off(warp * 16 + (lane & 15), 2 * kk + (lane >> 4));
            ldmatrix_x4(aq[0], aq[1], aq[2], aq[3], qs + ao);
            ldmatrix_x4(ad[0], ad[1], ad[2], ad[3], das + ao);
            ldmatrix_x4(al[0], al[1], al[2], al[3], dls + ao);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b0, b1, b2, b3;
                const uint32_t bo = tile_off(np * 16 + (lane >> 4) * 8 + (lane & 7), 2 * kk + ((lane >> 3) & 1));
                ldmatrix_x4(b0, b1, b2, b3, ks + bo);
                mma_bf16(s[2 * np], aq, b0, b1);
                mma_bf16(s[2 * np + 1], aq, b2, b3);
                ldmatrix_x4(b0, b1, b2, b3, vs + bo);
                mma_bf16(dp[2 * np], ad, b0, b1);
                mma_bf16(dp[2 * np + 1], ad, b2, b3);
                mma_bf16(dp[2 * np], al, b0, b1);
                mma_bf16(dp[2 * np + 1], al, b2, b3);
            }
        }
        // masked base-2 scores
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = kbase + nt * 8 + 2 * (lane & 3) + (e & 1);
                const int i = e < 2 ? r0 : r1;
                const bool vis = j <= i && j > i - L.W && j < L.S && i < L.S;
                s[nt][e] = vis ? s[nt][e] * L.scale_log2 : -INFINITY;
            }
        }
        if (pass == 0) {
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
                mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
            const float c0 = exp2f(m0 - mu0), c1 = exp2f(m1 - mu1);
            l0 *= c0; n0 *= c0; l1 *= c1; n1 *= c1;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float ev = exp2f(s[nt][e] - (e < 2 ? mu0 : mu1));
                    if (e < 2) { l0 += ev; n0 += ev * dp[nt][e]; } else { l1 += ev; n1 += ev * dp[nt][e]; }
                }
            }
            m0 = mn0; m1 = mn1;
            continue;
        }
        // pass 2: dS = P (dP - Delta), dQ~ += dS K~ as hi*hi + lo*hi + hi*lo
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pv = exp2f(s[nt][e] - (e < 2 ? lse0 : lse1));
                dp[nt][e] = pv * (dp[nt][e] - (e < 2 ? del0 : del1));
            }
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t ah[4], al[4];
            split_frag(dp, kk, ah, al);
#pragma unroll
            for (int dn = 0; dn < 8; ++dn) {
                uint32_t b0, b1, b2, b3;
                const uint32_t bo = tile_off(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * dn + (lane >> 4));
                ldmatrix_x4_trans(b0, b1, b2, b3, ks + bo);
                mma_bf16(dq[2 * dn], ah, b0, b1);
                mma_bf16(dq[2 * dn + 1], ah, b2, b3);
                mma_bf16(dq[2 * dn], al, b0, b1);
                mma_bf16(dq[2 * dn + 1], al, b2, b3);
                ldmatrix_x4_trans(b0, b1, b2, b3, kls + bo);
                mma_bf16(dq[2 * dn], ah, b0, b1);
                mma_bf16(dq[2 * dn + 1], ah, b2, b3);
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    if ((lane & 3) == 0) {
        const size_t base = ((size_t)b * L.Hq + h) * L.S;
        if (r0 < L.S) { p.delta[base + r0] = del0; p.lse2[base + r0] = lse0; }
        if (r1 < L.S) { p.delta[base + r1] = del1; p.lse2[base + r1] = lse1; }
    }
    // dQ~ (scaled) -> fp32 staging [64][128] in the K buffers
    float* stage = reinterpret_cast<float*>(sm.K[0]);
    const int lr0 = warp * 16 + (lane >> 2), lr1 = lr0 + 8;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        const int col = nt * 8 + 2 * (lane & 3);
        *reinterpret_cast<float2*>(stage + lr0 * kD + col) = make_float2(L.scale * dq[nt][0], L.scale * dq[nt][1]);
        *reinterpret_cast<float2*>(stage + lr1 * kD + col) = make_float2(L.scale * dq[nt][2], L.scale * dq[nt][3]);
    }
    __syncthreads();
    float dgacc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < 16; ++r) {
        const int row = warp * 16 + r, pos = q0 + row;
        if (pos >= L.S) break;
        const size_t off = ((size_t)(b * (size_t)L.S + pos) * L.Hq + h) * kD;
        uint2 raw = load_row4(L.q + off);
        float4 d4 = *reinterpret_cast<const float4*>(stage + row * kD + 4 * lane);
        float dy[4] = {d4.x, d4.y, d4.z, d4.w}, dx[4];
        prologue_row_backward(raw, gq4, L, pos, sm.ybuf[warp], dy, dx, dgacc);
        *reinterpret_cast<uint2*>(p.dq + off + 4 * lane) = make_uint2(pack_bf16(dx[0], dx[1]), pack_bf16(dx[2], dx[3]));
    }
    *reinterpret_cast<float4*>(&sm.dgq[warp][4 * lane]) = make_float4(dgacc[0], dgacc[1], dgacc[2], dgacc[3]);
    __syncthreads();
    if (tid < kD) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < DQ_THREADS / 32; ++w) t += sm.dgq[w][tid];
        p.dgq_part[(size_t)blockIdx.x * kD + tid] = t;
    }
}

// =====================================================================  bwd_main

constexpr int BM_KEYS = 64;     // keys per CTA (4 warps x 16)
constexpr int BM_Q = 64;        // queries per inner tile
constexpr int BM_THREADS = 128;

struct BwdMmaSmem {
    bf16 K[BM_KEYS * kD];     // K~ (normalised + rotated), swizzled rows
    bf16 V[BM_KEYS * kD];
    bf16 Q[BM_Q * kD];        // Q~ hi of the current query tile
    bf16 Ql[BM_Q * kD];       // Q~ lo
    bf16 dA[BM_Q * kD];
    bf16 dAl[BM_Q * kD];
    float lse2[BM_Q];         // base-2 log-sum-exp from bwd_dq
    float delta[BM_Q];
    float ybuf[BM_THREADS / 32][kD];
    float gq[kD], gk[kD];
    float dgk[BM_THREADS / 32][kD];
};

__global__ void __launch_bounds__(BM_THREADS, 1) bwd_main_kernel(const __grid_constant__ BwdParams p) {
    const LayerParams& L = p.L;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    BwdMmaSmem& sm = *reinterpret_cast<BwdMmaSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int nkt = (L.S + BM_KEYS - 1) / BM_KEYS;
    int bid = blockIdx.x;
    const int b = bid / (nkt * L.Hkv);
    bid -= b * nkt * L.Hkv;
    const int kvh = bid / nkt;
    const int kt = bid - kvh * nkt;  // low key tiles have the most work under full causal
    const int k0 = kt * BM_KEYS;

    if (tid < kD) {
        sm.gq[tid] = L.gamma_q[tid];
        sm.gk[tid] = L.gamma_k[tid];
    }
    __syncthreads();
    const float gq4[4] = {sm.gq[4 * lane], sm.gq[4 * lane + 1], sm.gq[4 * lane + 2], sm.gq[4 * lane + 3]};
    const float gk4[4] = {sm.gk[4 * lane], sm.gk[4 * lane + 1], sm.gk[4 * lane + 2], sm.gk[4 * lane + 3]};

    // ---- K~ and V for this CTA's 64 keys (warp w: rows 16w..16w+15)
    {
        uint2 raw[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            int pos = k0 + warp * 16 + r;
            raw[r] = pos < L.S ? load_row4(L.k + ((size_t)(b * (size_t)L.S + pos) * L.Hkv + kvh) * kD)
                               : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            int row = warp * 16 + r, pos = k0 + row;
            float y[4] = {0.f, 0.f, 0.f, 0.f};
            if (pos < L.S) prologue_row(raw[r], gk4, L, pos, sm.ybuf[warp], y);
            store_row_split(sm.K, nullptr, row, y);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int c = tid + BM_THREADS * i;
            int row = c >> 4, ch = c & 15, pos = k0 + row;
            bool ok = pos < L.S;
            const bf16* src = L.v + ((size_t)(b * (size_t)L.S + (ok ? pos : 0)) * L.Hkv + kvh) * kD + ch * 8;
            cp_async16(smem_u32(reinterpret_cast<char*>(sm.V) + tile_off(row, ch)), src, ok);
        }
        cp_async_commit();
    }

    float dk[16][4], dv[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;

    // this warp's keys: kw0 .. kw0+15; thread rows j0 = kw0 + lane/4, j1 = j0 + 8
    const int kw0 = k0 + warp * 16;
    const int j0 = kw0 + (lane >> 2), j1 = j0 + 8;
    const int qhi = min(L.S - 1, k0 + BM_KEYS - 1 + L.W - 1);
    const int qt_lo = k0 / BM_Q, qt_hi = qhi / BM_Q;

    for (int hh = 0; hh < L.G; ++hh) {
        const int h = kvh * L.G + hh;
        for (int qt = qt_lo; qt <= qt_hi; ++qt) {
            const int q0 = qt * BM_Q;
            __syncthreads();  // previous tile's readers of Q, dA are done
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int c = tid + BM_THREADS * i;
                int row = c >> 4, ch = c & 15, pos = q0 + row;
                bool ok = pos < L.S;
                const size_t go = ((size_t)(b * (size_t)L.S + (ok ? pos : 0)) * L.Hq + h) * kD + ch * 8;
                cp_async16(smem_u32(reinterpret_cast<char*>(sm.dA) + tile_off(row, ch)), p.dA + go, ok);
                cp_async16(smem_u32(reinterpret_cast<char*>(sm.dAl) + tile_off(row, ch)), p.dA_lo + go, ok);
            }
            cp_async_commit();
            if (tid < BM_Q) {
                int pos = q0 + tid;
                bool ok = pos < L.S;
                sm.lse2[tid] = ok ? p.lse2[((size_t)b * L.Hq + h) * L.S + pos] : INFINITY;
                sm.delta[tid] = ok ? p.delta[((size_t)b * L.Hq + h) * L.S + pos] : 0.f;
            }
            {
                uint2 raw[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    int pos = q0 + warp * 16 + r;
                    raw[r] = pos < L.S ? load_row4(L.q + ((size_t)(b * (size_t)L.S + pos) * L.Hq + h) * kD)
                                       : make_uint2(0u, 0u);
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    int row = warp * 16 + r, pos = q0 + row;
                    float y[4] = {0.f, 0.f, 0.f, 0.f};
                    if (pos < L.S) prologue_row(raw[r], gq4, L, pos, sm.ybuf[warp], y);
                    store_row_split(sm.Q, sm.Ql, row, y);
                }
            }
            cp_async_wait<0>();
            __syncthreads();

            // warp-level skip: keys [kw0, kw0+15] are seen by queries [kw0, kw0+15+W-1]
            const bool live = kw0 < L.S && q0 <= kw0 + 15 + L.W - 1 && q0 + BM_Q - 1 >= kw0;
            if (!live) continue;
            const uint32_t kb = smem_u32(sm.K), vb = smem_u32(sm.V), qb = smem_u32(sm.Q), qlb = smem_u32(sm.Ql),
                           db = smem_u32(sm.dA), dlb = smem_u32(sm.dAl);
            float st[8][4], dpt[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) st[i][e] = dpt[i][e] = 0.f;
            // S^T = K~ Q~^T and dP^T = V (dA_hi + dA_lo)^T  (16 keys x 64 queries)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t ak[4], av[4];
                const uint32_t ao = tile_off(warp * 16 + (lane & 15), 2 * kk + (lane >> 4));
                ldmatrix_x4(ak[0], ak[1], ak[2], ak[3], kb + ao);
                ldmatrix_x4(av[0], av[1], av[2], av[3], vb + ao);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    const uint32_t bo = tile_off(np * 16 + (lane >> 4) * 8 + (lane & 7), 2 * kk + ((lane >> 3) & 1));
                    ldmatrix_x4(b0, b1, b2, b3, qb + bo);
                    mma_bf16(st[2 * np], ak, b0, b1);
                    mma_bf16(st[2 * np + 1], ak, b2, b3);
                    ldmatrix_x4(b0, b1, b2, b3, db + bo);
                    mma_bf16(dpt[2 * np], av, b0, b1);
                    mma_bf16(dpt[2 * np + 1], av, b2, b3);
                    ldmatrix_x4(b0, b1, b2, b3, dlb + bo);
                    mma_bf16(dpt[2 * np], av, b0, b1);
                    mma_bf16(dpt[2 * np + 1], av, b2, b3);
                }
            }
            // P^T = exp2(S^T*scale*log2e - lse2), masked; dS^T = P^T (dP^T - Delta)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int ql = nt * 8 + 2 * (lane & 3) + (e & 1);
                    int i = q0 + ql;
                    int j = e < 2 ? j0 : j1;
                    bool vis = j <= i && j > i - L.W && i < L.S && j < L.S;
                    float pv = vis ? exp2f(st[nt][e] * L.scale_log2 - sm.lse2[ql]) : 0.f;
                    st[nt][e] = pv;
                    dpt[nt][e] = pv * (dpt[nt][e] - sm.delta[ql]);
                }
            }
            // dV += P^T dA ; dK~ += dS^T Q~   (hi*hi + lo*hi + hi*lo)
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                uint32_t ph[4], pl[4], sh[4], sl[4];
                split_frag(st, kq, ph, pl);
                split_frag(dpt, kq, sh, sl);
#pragma unroll
                for (int dn = 0; dn < 8; ++dn) {
                    uint32_t b0, b1, b2, b3;
                    const uint32_t bo = tile_off(16 * kq + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * dn + (lane >> 4));
                    ldmatrix_x4_trans(b0, b1, b2, b3, db + bo);
                    mma_bf16(dv[2 * dn], ph, b0, b1);
                    mma_bf16(dv[2 * dn + 1], ph, b2, b3);
                    mma_bf16(dv[2 * dn], pl, b0, b1);
                    mma_bf16(dv[2 * dn + 1], pl, b2, b3);
                    ldmatrix_x4_trans(b0, b1, b2, b3, dlb + bo);
                    mma_bf16(dv[2 * dn], ph, b0, b1);
                    mma_bf16(dv[2 * dn + 1], ph, b2, b3);
                    ldmatrix_x4_trans(b0, b1, b2, b3, qb + bo);
                    mma_bf16(dk[2 * dn], sh, b0, b1);
                    mma_bf16(dk[2 * dn + 1], sh, b2, b3);
                    mma_bf16(dk[2 * dn], sl, b0, b1);
                    mma_bf16(dk[2 * dn + 1], sl, b2, b3);
                    ldmatrix_x4_trans(b0, b1, b2, b3, qlb + bo);
                    mma_bf16(dk[2 * dn], sh, b0, b1);
                    mma_bf16(dk[2 * dn + 1], sh, b2, b3);
                }
            }
        }
    }

    // ---- epilogue: dv direct; dK~ -> stage -> RMSNorm/RoPE backward -> dk, d_gamma_k
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        const int col = nt * 8 + 2 * (lane & 3);
        if (j0 < L.S)
            *reinterpret_cast<uint32_t*>(p.dv + ((size_t)(b * (size_t)L.S + j0) * L.Hkv + kvh) * kD + col) = pack_bf16(dv[nt][0], dv[nt][1]);
        if (j1 < L.S)
            *reinterpret_cast<uint32_t*>(p.dv + ((size_t)(b * (size_t)L.S + j1) * L.Hkv + kvh) * kD + col) = pack_bf16(dv[nt][2], dv[nt][3]);
    }
    __syncthreads();
    float* stage = reinterpret_cast<float*>(sm.Q);  // Q + Ql = 32 KB = [64][128] fp32
    {
        const int rr0 = warp * 16 + (lane >> 2), rr1 = rr0 + 8;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int col = nt * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2*>(stage + rr0 * kD + col) = make_float2(dk[nt][0] * L.scale, dk[nt][1] * L.scale);
            *reinterpret_cast<float2*>(stage + rr1 * kD + col) = make_float2(dk[nt][2] * L.scale, dk[nt][3] * L.scale);
        }
    }
    __syncthreads();
    float dgacc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < 16; ++r) {
        const int row = warp * 16 + r, pos = k0 + row;
        if (pos >= L.S) break;
        const size_t off = ((size_t)(b * (size_t)L.S + pos) * L.Hkv + kvh) * kD;
        uint2 raw = load_row4(L.k + off);
        float4 d4 = *reinterpret_cast<const float4*>(stage + row * kD + 4 * lane);
        float dy[4] = {d4.x, d4.y, d4.z, d4.w}, dx[4];
        prologue_row_backward(raw, gk4, L, pos, sm.ybuf[warp], dy, dx, dgacc);
        *reinterpret_cast<uint2*>(p.dk + off + 4 * lane) = make_uint2(pack_bf16(dx[0], dx[1]), pack_bf16(dx[2], dx[3]));
    }
    *reinterpret_cast<float4*>(&sm.dgk[warp][4 * lane]) = make_float4(dgacc[0], dgacc[1], dgacc[2], dgacc[3]);
    __syncthreads();
    if (tid < kD) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < BM_THREADS / 32; ++w) s += sm.dgk[w][tid];
        p.dgk_part[(size_t)blockIdx.x * kD + tid] = s;
    }
}

// =====================================================================  d_gamma reduction

// 1024 threads: 8 groups of 128 sum parts p = group (mod 8) in increasing order; the group
// sums are then added in group order.  Fixed order -> bitwise reproducible.
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
        for (int g = 0; g < 8; ++g) t += acc[g][d];
        out[d] = t;
    }
}

// =====================================================================  host-side launch

int bwd_mma_n_k_parts(int B, int S, int Hkv) { return ((S + BM_KEYS - 1) / BM_KEYS) * Hkv * B; }
long long bwd_mma_n_q_parts(int B, int S, int Hq) {
    return (long long)((S + DQ_BM - 1) / DQ_BM) * Hq * B;
}

extern const char* const kBwdMmaKernelNames[] = {"bwd_pre_kernel", "bwd_dq_kernel", "bwd_main_kernel",
                                                 "dgamma_reduce_kernel(k)", "dgamma_reduce_kernel(q)"};
extern const int kBwdMmaKernelCount = 5;

namespace {
// records events[2i] before / events[2i+1] after kernel i when i < n_pairs
struct KernelEvents {
    void* const* ev;
    int n;
    cudaStream_t s;
    cudaError_t before(int i) const {
        return (i < n) ? cudaEventRecord(static_cast<cudaEvent_t>(ev[2 * i]), s) : cudaSuccess;
    }
    cudaError_t after(int i) const {
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return (i < n) ? cudaEventRecord(static_cast<cudaEvent_t>(ev[2 * i + 1]), s) : cudaSuccess;
    }
};
}  // namespace

cudaError_t launch_bwd_mma(const BwdParams& p, cudaStream_t stream, void* const* events, int n_pairs) {
    const LayerParams& L = p.L;
    const KernelEvents ke{events, n_pairs, stream};
    const long long nrows = (long long)L.B * L.S * L.Hq;
    const size_t smem_dq = sizeof(BwdDqSmem), smem_main = sizeof(BwdMmaSmem);
    cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dq);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(bwd_main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_main);
    if (e != cudaSuccess) return e;
    if ((e = ke.before(0)) != cudaSuccess) return e;
    bwd_pre_kernel<<<(unsigned)((nrows + PRE_WARPS - 1) / PRE_WARPS), PRE_WARPS * 32, 0, stream>>>(p);
    if ((e = ke.after(0)) != cudaSuccess) return e;
    if ((e = ke.before(1)) != cudaSuccess) return e;
    bwd_dq_kernel<<<(unsigned)p.n_q_parts, DQ_THREADS, smem_dq, stream>>>(p);
    if ((e = ke.after(1)) != cudaSuccess) return e;
    if ((e = ke.before(2)) != cudaSuccess) return e;
    bwd_main_kernel<<<(unsigned)p.n_k_parts, BM_THREADS, smem_main, stream>>>(p);
    if ((e = ke.after(2)) != cudaSuccess) return e;
    if ((e = ke.before(3)) != cudaSuccess) return e;
    dgamma_reduce_kernel<<<1, 1024, 0, stream>>>(p.dgk_part, p.n_k_parts, p.dgamma_k);
    if ((e = ke.after(3)) != cudaSuccess) return e;
    if ((e = ke.before(4)) != cudaSuccess) return e;
    dgamma_reduce_kernel<<<1, 1024, 0, stream>>>(p.dgq_part, p.n_q_parts, p.dgamma_q);
    return ke.after(4);
}

}  // namespace zgcm
