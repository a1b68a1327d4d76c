// fwd_mma.cu — gated window-attention forward on the warp-level tensor-core path
// (mma.sync m16n8k16 bf16 -> fp32).  Kept as the comparison baseline beside the
// tcgen05 kernels, and as the path for shapes those kernels do not take.
//
// One CTA = 128 query rows of one (batch, query head); 8 warps x 16 rows.  Key tiles of
// 64 rows are visited only where the window [i-W+1, i] of some row in the CTA reaches
// them, and a warp skips a tile that no row of its 16 can see.
//
// Steps (ZGCM-1 layer; see common.cuh for the page citations):
//   prologue  q, k rows -> RMSNorm(gamma) -> partial RoPE -> bf16 in shared memory
//   scores    S = scale * Q K^T, masked to i-W < j <= i
//   softmax   online, fp32, base-2 exponent with scale*log2(e) folded in
//   P.V       O += P V
//   epilogue  out = sigmoid(g) * O / l   (rounded once to bf16);  lse = ln sum exp
#include "common.cuh"

namespace zgcm {

constexpr int FM_BM = 128;
constexpr int FM_BN = 64;
constexpr int FM_THREADS = 256;

struct FwdMmaSmem {
    bf16 Q[FM_BM * kD];          // 32 KB, swizzled rows (tile_off)
    bf16 K[2][FM_BN * kD];       // 2 x 16 KB
    bf16 V[2][FM_BN * kD];       // 2 x 16 KB
    float ybuf[FM_THREADS / 32][kD];
    float gq[kD], gk[kD];
};
// the epilogue reuses Q..V (96 KB) as a [128][132] fp32 staging tile
static_assert(FM_BM * 132 * 4 <= sizeof(bf16) * (FM_BM * kD + 4 * FM_BN * kD), "staging fits");

__device__ __forceinline__ void fm_store_row(bf16* tile, int row, const float y[4]) {
    const int lane = threadIdx.x & 31;
    uint2 u = make_uint2(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]));
    *reinterpret_cast<uint2*>(reinterpret_cast<char*>(tile) + tile_off(row, lane >> 1) + (lane & 1) * 8) = u;
}

// K prologue (8 rows per warp) + V via cp.async for key tile starting at kbase.
__device__ __forceinline__ void fm_load_kv(const LayerParams& L, FwdMmaSmem& sm, int buf, int b,
                                           int kvh, int kbase) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // V: 64 rows x 16 chunks of 16 B
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int c = tid + FM_THREADS * i;
        int row = c >> 4, ch = c & 15;
        int pos = kbase + row;
        bool ok = pos < L.S;
        const bf16* src = L.v + ((size_t)(b * (size_t)L.S + (ok ? pos : 0)) * L.Hkv + kvh) * kD + ch * 8;
        cp_async16(smem_u32(reinterpret_cast<char*>(sm.V[buf]) + tile_off(row, ch)), src, ok);
    }
    cp_async_commit();
    // K: normalise + rotate
    uint2 raw[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int pos = kbase + warp * 8 + r;
        raw[r] = pos < L.S ? load_row4(L.k + ((size_t)(b * (size_t)L.S + pos) * L.Hkv + kvh) * kD)
                           : make_uint2(0u, 0u);
    }
    float g4[4] = {sm.gk[4 * lane], sm.gk[4 * lane + 1], sm.gk[4 * lane + 2], sm.gk[4 * lane + 3]};
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int row = warp * 8 + r, pos = kbase + row;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
        if (pos < L.S) prologue_row(raw[r], g4, L, pos, sm.ybuf[warp], y);
        fm_store_row(sm.K[buf], row, y);
    }
}

__global__ void __launch_bounds__(FM_THREADS, 1) fwd_mma_kernel(const __grid_constant__ FwdParams p) {
    const LayerParams& L = p.L;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    FwdMmaSmem& sm = *reinterpret_cast<FwdMmaSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int nqt = (L.S + FM_BM - 1) / FM_BM;
    int bid = blockIdx.x;
    const int b = bid / (nqt * L.Hq);
    bid -= b * nqt * L.Hq;
    const int h = bid / nqt;
    int qt = bid - h * nqt;
    if (L.W >= L.S) qt = nqt - 1 - qt;  // full causal: longest rows first
    const int kvh = h / L.G;
    const int q0 = qt * FM_BM;

    if (tid < kD) {
        sm.gq[tid] = L.gamma_q[tid];
        sm.gk[tid] = L.gamma_k[tid];
    }
    __syncthreads();

    // ---- Q prologue: warp w -> rows 16w .. 16w+15
    {
        uint2 raw[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            int pos = q0 + warp * 16 + r;
            raw[r] = pos < L.S ? load_row4(L.q + ((size_t)(b * (size_t)L.S + pos) * L.Hq + h) * kD)
                               : make_uint2(0u, 0u);
        }
        float g4[4] = {sm.gq[4 * lane], sm.gq[4 * lane + 1], sm.gq[4 * lane + 2], sm.gq[4 * lane + 3]};
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            int row = warp * 16 + r, pos = q0 + row;
            float y[4] = {0.f, 0.f, 0.f, 0.f};
            if (pos < L.S) prologue_row(raw[r], g4, L, pos, sm.ybuf[warp], y);
            fm_store_row(sm.Q, row, y);
        }
    }

    const int klo = max(0, q0 - L.W + 1);
    const int khi = min(L.S - 1, q0 + FM_BM - 1);
    const int kt_lo = klo / FM_BN, kt_hi = khi / FM_BN;

    // per-thread rows: r0 = q0 + 16*warp + lane/4, r1 = r0 + 8
    const int wq0 = q0 + warp * 16;
    const int r0 = wq0 + (lane >> 2), r1 = r0 + 8;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    fm_load_kv(L, sm, 0, b, kvh, kt_lo * FM_BN);

    for (int kt = kt_lo; kt <= kt_hi; ++kt) {
        const int buf = (kt - kt_lo) & 1;
        cp_async_wait<0>();
        __syncthreads();
        if (kt < kt_hi) fm_load_kv(L, sm, buf ^ 1, b, kvh, (kt + 1) * FM_BN);
        const int kbase = kt * FM_BN;
        // warp-level skip: rows [wq0, wq0+15] see keys [wq0-W+1, wq0+15]
        const bool live = wq0 < L.S && kbase <= wq0 + 15 && kbase + FM_BN - 1 >= wq0 - L.W + 1;
        if (live) {
            float s[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
            const uint32_t qbase = smem_u32(sm.Q), kb = smem_u32(sm.K[buf]), vb = smem_u32(sm.V[buf]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t a[4];
                ldmatrix_x4(a[0], a[1], a[2], a[3], qbase + tile_off(warp * 16 + (lane & 15), 2 * kk + (lane >> 4)));
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(b0, b1, b2, b3,
                                kb + tile_off(np * 16 + (lane >> 4) * 8 + (lane & 7), 2 * kk + ((lane >> 3) & 1)));
                    mma_bf16(s[2 * np], a, b0, b1);
                    mma_bf16(s[2 * np + 1], a, b2, b3);
                }
            }
            // mask + online softmax (base 2)
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int j = kbase + nt * 8 + 2 * (lane & 3) + (e & 1);
                    int i = e < 2 ? r0 : r1;
                    bool vis = j <= i && j > i - L.W && j < L.S;
                    float x = vis ? s[nt][e] * L.scale_log2 : -INFINITY;
                    s[nt][e] = x;
                    if (e < 2) mx0 = fmaxf(mx0, x); else mx1 = fmaxf(mx1, x);
                }
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
            const float c0 = exp2f(m0 - mu0), c1 = exp2f(m1 - mu1);
            m0 = mn0; m1 = mn1;
            float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                s[nt][0] = exp2f(s[nt][0] - mu0);
                s[nt][1] = exp2f(s[nt][1] - mu0);
                s[nt][2] = exp2f(s[nt][2] - mu1);
                s[nt][3] = exp2f(s[nt][3] - mu1);
                ps0 += s[nt][0] + s[nt][1];
                ps1 += s[nt][2] + s[nt][3];
            }
            l0 = l0 * c0 + ps0;
            l1 = l1 * c1 + ps1;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                o[i][0] *= c0; o[i][1] *= c0;
                o[i][2] *= c1; o[i][3] *= c1;
            }
            // O += P V
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a[4];
                a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
                for (int dn = 0; dn < 8; ++dn) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(b0, b1, b2, b3,
                                      vb + tile_off(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * dn + (lane >> 4)));
                    mma_bf16(o[2 * dn], a, b0, b1);
                    mma_bf16(o[2 * dn + 1], a, b2, b3);
                }
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- finish rows: l over the quad, lse, normalise
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
    if ((lane & 3) == 0) {
        if (r0 < L.S) p.lse[((size_t)b * L.Hq + h) * L.S + r0] = (m0 + log2f(l0)) * kLn2;
        if (r1 < L.S) p.lse[((size_t)b * L.Hq + h) * L.S + r1] = (m1 + log2f(l1)) * kLn2;
    }
    float* stage = reinterpret_cast<float*>(smem_raw);  // [128][132]
    {
        const int rr0 = warp * 16 + (lane >> 2), rr1 = rr0 + 8;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            int col = nt * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2*>(stage + rr0 * 132 + col) = make_float2(o[nt][0] * inv0, o[nt][1] * inv0);
            *reinterpret_cast<float2*>(stage + rr1 * 132 + col) = make_float2(o[nt][2] * inv1, o[nt][3] * inv1);
        }
    }
    __syncthreads();
    // ---- gate epilogue: 8 elements per step, 16 threads per 256-byte row
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        int c = tid + FM_THREADS * it;
        int row = c >> 4, col = (c & 15) * 8;
        int pos = q0 + row;
        if (pos >= L.S) continue;
        size_t off = ((size_t)(b * (size_t)L.S + pos) * L.Hq + h) * kD + col;
        uint4 gr = *reinterpret_cast<const uint4*>(L.g + off);
        const float* a = stage + row * 132 + col;
        float2 g0 = unpack_bf16(gr.x), g1 = unpack_bf16(gr.y), g2 = unpack_bf16(gr.z), g3 = unpack_bf16(gr.w);
        uint4 ov;
        ov.x = pack_bf16(sigmoidf_(g0.x) * a[0], sigmoidf_(g0.y) * a[1]);
        ov.y = pack_bf16(sigmoidf_(g1.x) * a[2], sigmoidf_(g1.y) * a[3]);
        ov.z = pack_bf16(sigmoidf_(g2.x) * a[4], sigmoidf_(g2.y) * a[5]);
        ov.w = pack_bf16(sigmoidf_(g3.x) * a[6], sigmoidf_(g3.y) * a[7]);
        *reinterpret_cast<uint4*>(p.out + off) = ov;
    }
}

size_t fwd_mma_smem_bytes() { return sizeof(FwdMmaSmem); }

cudaError_t launch_fwd_mma(const FwdParams& p, cudaStream_t stream) {
    const size_t smem = sizeof(FwdMmaSmem);
    cudaError_t e = cudaFuncSetAttribute(fwd_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nqt = (p.L.S + FM_BM - 1) / FM_BM;
    const long long grid = nqt * p.L.Hq * (long long)p.L.B;
    fwd_mma_kernel<<<(unsigned)grid, FM_THREADS, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace zgcm
