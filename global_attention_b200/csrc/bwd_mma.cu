// bwd_mma.cu — gated window-attention backward on the warp-level tensor-core path
// (mma.sync m16n8k16 bf16 -> fp32).  Exact gradients of L = sum(dout * out) for the
// ZGCM-1 layer (definition and page citations in common.cuh).
//
// Kernels, in launch order:
//   bwd_pre     per (b, s, h) row: Delta = sum_d dout*out; dg = dout*out*(1-sigmoid(g));
//               dA = dout*sigmoid(g)   (out = sigmoid(g)*A, so neither needs A itself)
//   bwd_main    per (b, KV head, 64-key tile), over the Hq/Hkv query heads of the group and
//               every 64-query tile whose window reaches the keys:
//                 P^T = exp(S^T - lse), dV += P^T dA, dP^T = V dA^T, dS^T = P^T (dP^T - Delta),
//                 dK~ += dS^T Q~, dQ~ += dS K~ (fp32 atomics into the workspace);
//               epilogue: dk = RMSNorm/RoPE backward of scale*dK~, dv, d_gamma_k partials
//   bwd_dq      per row: dq = RMSNorm/RoPE backward of scale*dQ~, d_gamma_q partials
//   dgamma      fixed-order sum of the partials (deterministic)
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
    float delta = 0.f, dgv[4], dav[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float sg = sigmoidf_(g[e]);
        delta += d[e] * o[e];
        dgv[e] = d[e] * o[e] * (1.f - sg);
        dav[e] = d[e] * sg;
    }
    delta = warp_sum(delta);
    *reinterpret_cast<uint2*>(p.dg + off) = make_uint2(pack_bf16(dgv[0], dgv[1]), pack_bf16(dgv[2], dgv[3]));
    *reinterpret_cast<uint2*>(p.dA + off) = make_uint2(pack_bf16(dav[0], dav[1]), pack_bf16(dav[2], dav[3]));
    if (lane == 0) {
        const long long h = row % L.Hq, bs = row / L.Hq, s = bs % L.S, b = bs / L.S;
        p.delta[((size_t)b * L.Hq + h) * L.S + s] = delta;
    }
}

// =====================================================================  bwd_main

constexpr int BM_KEYS = 64;     // keys per CTA (4 warps x 16)
constexpr int BM_Q = 64;        // queries per inner tile
constexpr int BM_THREADS = 128;

struct BwdMmaSmem {
    bf16 K[BM_KEYS * kD];     // K~ (normalised + rotated), swizzled rows
    bf16 V[BM_KEYS * kD];
    bf16 Q[BM_Q * kD];        // Q~ of the current query tile
    bf16 dA[BM_Q * kD];
    bf16 dS[BM_KEYS * BM_Q];  // [key][query], 128-byte rows, chunk ^= row & 7
    float lse2[BM_Q];         // lse * log2(e)
    float delta[BM_Q];
    float ybuf[BM_THREADS / 32][kD];
    float gq[kD], gk[kD];
    float dgk[BM_THREADS / 32][kD];
};

__device__ __forceinline__ uint32_t ds_off(int row, int chunk) {
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void bm_store_row(bf16* tile, int row, const float y[4]) {
    const int lane = threadIdx.x & 31;
    uint2 u = make_uint2(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]));
    *reinterpret_cast<uint2*>(reinterpret_cast<char*>(tile) + tile_off(row, lane >> 1) + (lane & 1) * 8) = u;
}

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
            bm_store_row(sm.K, row, y);
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
            __syncthreads();  // previous tile's readers of Q, dA, dS are done
            // dA tile (cp.async), Q~ tile (prologue), lse, Delta
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int c = tid + BM_THREADS * i;
                int row = c >> 4, ch = c & 15, pos = q0 + row;
                bool ok = pos < L.S;
                const bf16* src = p.dA + ((size_t)(b * (size_t)L.S + (ok ? pos : 0)) * L.Hq + h) * kD + ch * 8;
                cp_async16(smem_u32(reinterpret_cast<char*>(sm.dA) + tile_off(row, ch)), src, ok);
            }
            cp_async_commit();
            if (tid < BM_Q) {
                int pos = q0 + tid;
                bool ok = pos < L.S;
                sm.lse2[tid] = ok ? p.lse[((size_t)b * L.Hq + h) * L.S + pos] * kLog2e : INFINITY;
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
                    bm_store_row(sm.Q, row, y);
                }
            }
            cp_async_wait<0>();
            __syncthreads();

            // warp-level skip: keys [kw0, kw0+15] are seen by queries [kw0, kw0+15+W-1]
            const bool live = kw0 < L.S && q0 <= kw0 + 15 + L.W - 1 && q0 + BM_Q - 1 >= kw0;
            const uint32_t kb = smem_u32(sm.K), vb = smem_u32(sm.V), qb = smem_u32(sm.Q), db = smem_u32(sm.dA);
            if (live) {
                float st[8][4], dpt[8][4];
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int e = 0; e < 4; ++e) st[i][e] = dpt[i][e] = 0.f;
                // S^T = K~ Q~^T and dP^T = V dA^T  (16 keys x 64 queries)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint32_t ak[4], av[4];
                    ldmatrix_x4(ak[0], ak[1], ak[2], ak[3], kb + tile_off(warp * 16 + (lane & 15), 2 * kk + (lane >> 4)));
                    ldmatrix_x4(av[0], av[1], av[2], av[3], vb + tile_off(warp * 16 + (lane & 15), 2 * kk + (lane >> 4)));
#pragma unroll
                    for (int np = 0; np < 4; ++np) {
                        uint32_t b0, b1, b2, b3;
                        const int rr = np * 16 + (lane >> 4) * 8 + (lane & 7), cc = 2 * kk + ((lane >> 3) & 1);
                        ldmatrix_x4(b0, b1, b2, b3, qb + tile_off(rr, cc));
                        mma_bf16(st[2 * np], ak, b0, b1);
                        mma_bf16(st[2 * np + 1], ak, b2, b3);
                        ldmatrix_x4(b0, b1, b2, b3, db + tile_off(rr, cc));
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
                // dV += P^T dA ; dK~ += dS^T Q~   (A from registers, B via ldmatrix.trans)
#pragma unroll
                for (int kq = 0; kq < 4; ++kq) {
                    uint32_t ap[4], as[4];
                    ap[0] = pack_bf16(st[2 * kq][0], st[2 * kq][1]);
                    ap[1] = pack_bf16(st[2 * kq][2], st[2 * kq][3]);
                    ap[2] = pack_bf16(st[2 * kq + 1][0], st[2 * kq + 1][1]);
                    ap[3] = pack_bf16(st[2 * kq + 1][2], st[2 * kq + 1][3]);
                    as[0] = pack_bf16(dpt[2 * kq][0], dpt[2 * kq][1]);
                    as[1] = pack_bf16(dpt[2 * kq][2], dpt[2 * kq][3]);
                    as[2] = pack_bf16(dpt[2 * kq + 1][0], dpt[2 * kq + 1][1]);
                    as[3] = pack_bf16(dpt[2 * kq + 1][2], dpt[2 * kq + 1][3]);
#pragma unroll
                    for (int dn = 0; dn < 8; ++dn) {
                        uint32_t b0, b1, b2, b3;
                        const int rr = 16 * kq + (lane & 7) + ((lane >> 3) & 1) * 8, cc = 2 * dn + (lane >> 4);
                        ldmatrix_x4_trans(b0, b1, b2, b3, db + tile_off(rr, cc));
                        mma_bf16(dv[2 * dn], ap, b0, b1);
                        mma_bf16(dv[2 * dn + 1], ap, b2, b3);
                        ldmatrix_x4_trans(b0, b1, b2, b3, qb + tile_off(rr, cc));
                        mma_bf16(dk[2 * dn], as, b0, b1);
                        mma_bf16(dk[2 * dn + 1], as, b2, b3);
                    }
                    // dS^T to shared memory ([key][query], bf16) for the dQ product
                    char* dsb = reinterpret_cast<char*>(sm.dS);
                    const int kr0 = warp * 16 + (lane >> 2), kr1 = kr0 + 8;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int nt = 2 * kq + half;
                        const int ql = nt * 8 + 2 * (lane & 3);
                        *reinterpret_cast<uint32_t*>(dsb + ds_off(kr0, ql >> 3) + (ql & 7) * 2) = as[2 * half];
                        *reinterpret_cast<uint32_t*>(dsb + ds_off(kr1, ql >> 3) + (ql & 7) * 2) = as[2 * half + 1];
                    }
                }
            } else {
                // zero this warp's dS^T rows so the dQ product reads no stale values
                char* dsb = reinterpret_cast<char*>(sm.dS);
                for (int c = lane; c < 16 * 8; c += 32) {
                    int row = warp * 16 + (c >> 3), ch = c & 7;
                    *reinterpret_cast<uint4*>(dsb + ds_off(row, ch)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            __syncthreads();
            // dQ~ (64 queries x 128) += dS (64 x 64 keys) K~ (64 x 128); warp w: queries 16w..16w+15,
            // in four 32-column slices to bound the live accumulator registers
            const int qr0 = q0 + warp * 16 + (lane >> 2), qr1 = qr0 + 8;
            const uint32_t dsb = smem_u32(sm.dS);
            if (q0 + warp * 16 < L.S) {
#pragma unroll
                for (int dc = 0; dc < 4; ++dc) {
                    float acc[4][4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        uint32_t a[4];
                        ldmatrix_x4_trans(a[0], a[1], a[2], a[3],
                                          dsb + ds_off(16 * kk + (lane & 7) + (lane >> 4) * 8, 2 * warp + ((lane >> 3) & 1)));
#pragma unroll
                        for (int dn = 0; dn < 2; ++dn) {
                            uint32_t b0, b1, b2, b3;
                            ldmatrix_x4_trans(b0, b1, b2, b3,
                                              kb + tile_off(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8, 4 * dc + 2 * dn + (lane >> 4)));
                            mma_bf16(acc[2 * dn], a, b0, b1);
                            mma_bf16(acc[2 * dn + 1], a, b2, b3);
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        const int col = 32 * dc + 8 * nt + 2 * (lane & 3);
                        if (qr0 < L.S)
                            atomicAdd(reinterpret_cast<float2*>(p.dq_acc + ((size_t)(b * (size_t)L.S + qr0) * L.Hq + h) * kD + col),
                                      make_float2(acc[nt][0], acc[nt][1]));
                        if (qr1 < L.S)
                            atomicAdd(reinterpret_cast<float2*>(p.dq_acc + ((size_t)(b * (size_t)L.S + qr1) * L.Hq + h) * kD + col),
                                      make_float2(acc[nt][2], acc[nt][3]));
                    }
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
    float* stage = reinterpret_cast<float*>(sm.Q);  // Q + dA = 32 KB = [64][128] fp32
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

// =====================================================================  bwd_dq

constexpr int DQ_WARPS = 8;
constexpr int DQ_ROWS_PER_WARP = 32;

__global__ void __launch_bounds__(DQ_WARPS * 32) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
    const LayerParams& L = p.L;
    __shared__ float ybuf[DQ_WARPS][kD];
    __shared__ float dgq[DQ_WARPS][kD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long nrows = (long long)L.B * L.S * L.Hq;
    const float g4[4] = {L.gamma_q[4 * lane], L.gamma_q[4 * lane + 1], L.gamma_q[4 * lane + 2], L.gamma_q[4 * lane + 3]};
    float dgacc[4] = {0.f, 0.f, 0.f, 0.f};
    const long long first = ((long long)blockIdx.x * DQ_WARPS + warp) * DQ_ROWS_PER_WARP;
    for (int r = 0; r < DQ_ROWS_PER_WARP; ++r) {
        const long long row = first + r;
        if (row >= nrows) break;
        const int pos = (int)((row / L.Hq) % L.S);
        const size_t off = (size_t)row * kD;
        uint2 raw = load_row4(L.q + off);
        float4 a = *reinterpret_cast<const float4*>(p.dq_acc + off + 4 * lane);
        float dy[4] = {a.x * L.scale, a.y * L.scale, a.z * L.scale, a.w * L.scale}, dx[4];
        prologue_row_backward(raw, g4, L, pos, ybuf[warp], dy, dx, dgacc);
        *reinterpret_cast<uint2*>(p.dq + off + 4 * lane) = make_uint2(pack_bf16(dx[0], dx[1]), pack_bf16(dx[2], dx[3]));
    }
    *reinterpret_cast<float4*>(&dgq[warp][4 * lane]) = make_float4(dgacc[0], dgacc[1], dgacc[2], dgacc[3]);
    __syncthreads();
    if (threadIdx.x < kD) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < DQ_WARPS; ++w) s += dgq[w][threadIdx.x];
        p.dgq_part[(size_t)blockIdx.x * kD + threadIdx.x] = s;
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
    const long long rows = (long long)B * S * Hq, per = (long long)DQ_WARPS * DQ_ROWS_PER_WARP;
    return (rows + per - 1) / per;
}

cudaError_t launch_bwd_mma(const BwdParams& p, cudaStream_t stream, cudaEvent_t ev0, cudaEvent_t ev1) {
    const LayerParams& L = p.L;
    const long long nrows = (long long)L.B * L.S * L.Hq;
    cudaError_t e = cudaMemsetAsync(p.dq_acc, 0, (size_t)nrows * kD * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    bwd_pre_kernel<<<(unsigned)((nrows + PRE_WARPS - 1) / PRE_WARPS), PRE_WARPS * 32, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t smem = sizeof(BwdMmaSmem);
    e = cudaFuncSetAttribute(bwd_main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (ev0 && (e = cudaEventRecord(ev0, stream)) != cudaSuccess) return e;
    bwd_main_kernel<<<(unsigned)p.n_k_parts, BM_THREADS, smem, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev1 && (e = cudaEventRecord(ev1, stream)) != cudaSuccess) return e;
    bwd_dq_kernel<<<(unsigned)p.n_q_parts, DQ_WARPS * 32, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    dgamma_reduce_kernel<<<1, 1024, 0, stream>>>(p.dgk_part, p.n_k_parts, p.dgamma_k);
    dgamma_reduce_kernel<<<1, 1024, 0, stream>>>(p.dgq_part, p.n_q_parts, p.dgamma_q);
    return cudaGetLastError();
}

}  // namespace zgcm
