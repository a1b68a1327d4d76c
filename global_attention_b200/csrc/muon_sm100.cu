// muon_sm100.cu — the Muon optimiser step of one matrix parameter on tcgen05 / TMEM / TMA
// (sm_100a): momentum, scaling by a bound on the spectral norm, Newton–Schulz iterations,
// decoupled weight decay.
//
// What is computed (ZGCM-1 summary, section "前置知识 / Muon 优化器"; shibing624 review,
// section "⚙️ 训练系统": momentum 0.9, spectral-norm scaling, five Newton–Schulz steps,
// lr 2e-4, weight decay 0.1; readings where the pages are silent in include/zgcm_muon.h):
//   M  <- mu M + G                                    (fp32 momentum, bf16 gradient)
//   X0  = M / (||M||_F + eps)   on the wide orientation (X0 = M^T / .. for a tall M), bf16
//   X  <- a X + (b A + c A A) X,   A = X X^T          `steps` times, bf16 operands, fp32 sums
//   W  <- W (1 - lr wd) - lr X^(T)                    (fp32 master weights)
//
// Products: the library's tcgen05 GEMM (gemm_sm100.cu), C = alpha A op(B) + beta D (bf16 in
// and out, fp32 accumulation in TMEM): B is [N, K] for X X^T and A A (A symmetric: only the
// upper tiles, then mirrored) and [K, N] for (.) X.  The elementwise steps
// (momentum with the sum of squares, the scaling with the optional transpose, the update)
// are plain streaming kernels; the norm is summed in a fixed order, so a step is
// reproducible bit for bit.
#include <cudaTypedefs.h>

#include "zgcm_muon.h"
#include "gemm_sm100.cuh"
#include "sm100.cuh"

namespace zgcm {
int* library_error_word();  // zgcm_attn.cu: the site of an expired bounded wait

using namespace sm100;

namespace muon {

constexpr int RED_THREADS = 256;
constexpr int RED_BLOCKS = 296;              // partial sums of squares (2 blocks per SM)

// ------------------------------------------------------------------ elementwise kernels

// Block sum of `v` over RED_THREADS threads (fixed tree order); the total is in thread 0.
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x == 0)
        for (int w = 0; w < RED_THREADS / 32; ++w) t += red[w];
    return t;
}

// M <- mu M + G (n elements, n a multiple of 8) and each block's sum of squares of the new M
// (grid-stride over 8-element chunks; the grid is fixed, so the partition and every sum are too)
__global__ void __launch_bounds__(RED_THREADS) muon_momentum_kernel(float* __restrict__ M,
                                                                    const bf16* __restrict__ G, long long n,
                                                                    float mu, float* __restrict__ part) {
    __shared__ float red[RED_THREADS / 32];
    float ss = 0.f;
    const long long chunks = n / 8;
    for (long long i = (long long)blockIdx.x * RED_THREADS + threadIdx.x; i < chunks;
         i += (long long)gridDim.x * RED_THREADS) {
        const uint4 g = __ldg(reinterpret_cast<const uint4*>(G) + i);
        float4* mp = reinterpret_cast<float4*>(M) + 2 * i;
        float4 m0 = mp[0], m1 = mp[1];
        const float2 g0 = unpack_bf16(g.x), g1 = unpack_bf16(g.y), g2 = unpack_bf16(g.z), g3 = unpack_bf16(g.w);
        m0 = make_float4(fmaf(mu, m0.x, g0.x), fmaf(mu, m0.y, g0.y), fmaf(mu, m0.z, g1.x), fmaf(mu, m0.w, g1.y));
        m1 = make_float4(fmaf(mu, m1.x, g2.x), fmaf(mu, m1.y, g2.y), fmaf(mu, m1.z, g3.x), fmaf(mu, m1.w, g3.y));
        mp[0] = m0;
        mp[1] = m1;
        ss = fmaf(m0.x, m0.x, fmaf(m0.y, m0.y, fmaf(m0.z, m0.z, fmaf(m0.w, m0.w, ss))));
        ss = fmaf(m1.x, m1.x, fmaf(m1.y, m1.y, fmaf(m1.z, m1.z, fmaf(m1.w, m1.w, ss))));
    }
    const float t = block_sum(ss, red);
    if (threadIdx.x == 0) part[blockIdx.x] = t;
}

// Each block's sum of squares of a bf16 matrix (n elements, a multiple of 8)
__global__ void __launch_bounds__(RED_THREADS) muon_sumsq_kernel(const bf16* __restrict__ X, long long n,
                                                                 float* __restrict__ part) {
    __shared__ float red[RED_THREADS / 32];
    float ss = 0.f;
    const long long chunks = n / 8;
    for (long long i = (long long)blockIdx.x * RED_THREADS + threadIdx.x; i < chunks;
         i += (long long)gridDim.x * RED_THREADS) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(X) + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16(w[e]);
            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
        }
    }
    const float t = block_sum(ss, red);
    if (threadIdx.x == 0) part[blockIdx.x] = t;
}

// part[RED_BLOCKS] = 1 / (||.||_F + eps) from the RED_BLOCKS partial sums, added in one fixed
// order (one warp: lane l takes every 32nd partial, then a fixed tree)
__global__ void __launch_bounds__(32) muon_inv_norm_kernel(float* __restrict__ part, float eps) {
    float t = 0.f;
    for (int i = threadIdx.x; i < RED_BLOCKS; i += 32) t += part[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) part[RED_BLOCKS] = 1.0f / (sqrtf(t) + eps);
}

// dst = bf16(src * scale) for an m x n source, written as is ([m, n]) or transposed ([n, m]);
// fp32 or bf16 source.  scale = *inv (1 / (||src||_F + eps)) when given, else 1.
// 32 x 32 tiles through shared memory, blocks of 32 x 8 threads.
template <class T>
__global__ void __launch_bounds__(256) muon_scale_kernel(const T* __restrict__ src, bf16* __restrict__ dst, int m,
                                                         int n, int transpose, const float* __restrict__ inv_p) {
    __shared__ float tile[32][33];
    __shared__ float s_inv;
    if (threadIdx.x == 0 && threadIdx.y == 0) s_inv = inv_p ? *inv_p : 1.0f;
    const int i0 = (int)blockIdx.y * 32, j0 = (int)blockIdx.x * 32;
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int i = i0 + y, j = j0 + threadIdx.x;
        float x = 0.f;
        if (i < m && j < n) {
            if constexpr (sizeof(T) == 4)
                x = src[(size_t)i * n + j];
            else
                x = __bfloat162float(src[(size_t)i * n + j]);
        }
        tile[y][threadIdx.x] = x;
    }
    __syncthreads();
    const float inv = s_inv;
    for (int y = threadIdx.y; y < 32; y += 8) {
        if (transpose) {
            const int i = j0 + y, j = i0 + threadIdx.x;  // dst [n, m]
            if (i < n && j < m) dst[(size_t)i * m + j] = __float2bfloat16_rn(tile[threadIdx.x][y] * inv);
        } else {
            const int i = i0 + y, j = j0 + threadIdx.x;
            if (i < m && j < n) dst[(size_t)i * n + j] = __float2bfloat16_rn(tile[y][threadIdx.x] * inv);
        }
    }
}

// W <- W (1 - lr wd) - lr O for an m x n W; O = X ([m, n]) or X^T (X is [n, m] when transposed)
__global__ void __launch_bounds__(256) muon_update_kernel(float* __restrict__ W, const bf16* __restrict__ X, int m,
                                                          int n, int transposed, float lr, float wd) {
    __shared__ float tile[32][33];
    const int i0 = (int)blockIdx.y * 32, j0 = (int)blockIdx.x * 32;
    if (transposed) {
        for (int y = threadIdx.y; y < 32; y += 8) {
            const int r = j0 + y, cc = i0 + threadIdx.x;  // X [n, m]: row r (a column of W), col cc
            tile[y][threadIdx.x] = (r < n && cc < m) ? __bfloat162float(X[(size_t)r * m + cc]) : 0.f;
        }
        __syncthreads();
    }
    const float keep = 1.0f - lr * wd;
    for (int y = threadIdx.y; y < 32; y += 8) {
        const int i = i0 + y, j = j0 + threadIdx.x;
        if (i < m && j < n) {
            const float o = transposed ? tile[threadIdx.x][y] : __bfloat162float(X[(size_t)i * n + j]);
            float* w = W + (size_t)i * n + j;
            *w = fmaf(-lr, o, *w * keep);
        }
    }
}

// ------------------------------------------------------------------ host side

// C [M, N] = alpha A op(B) + beta D: A [M, K]; B [K, N] (b_kn) or [N, K]
cudaError_t launch_gemm(const bf16* A, const bf16* B, const bf16* D, bf16* C, int M, int N, int K, float alpha,
                        float beta, bool b_kn, cudaStream_t stream, bool upper = false) {
    GemmDesc g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.a[0] = GemmSeg{A, M, K, 0};
    g.b_kn = b_kn ? 1 : 0;
    g.b = B;
    g.c[0] = C;
    g.c_ld[0] = N;
    g.d = D;
    g.alpha = alpha;
    g.beta = beta;
    g.upper = upper;
    return zgcm::launch_gemm(g, library_error_word(), stream);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// workspace: two X buffers [p, q] and A, B buffers [p, p] (bf16), the partial sums
struct Ws {
    bf16 *x0, *x1, *a, *b;
    float* part;
};
size_t ws_layout(int m, int n, char* base, Ws* w) {
    const size_t p = (size_t)(m < n ? m : n), q = (size_t)(m < n ? n : m);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char* r = base + off;
        off = align256(off + bytes);
        return r;
    };
    char* x0 = take(p * q * 2);
    char* x1 = take(p * q * 2);
    char* a = take(p * p * 2);
    char* b = take(p * p * 2);
    char* part = take((RED_BLOCKS + 1) * sizeof(float));  // partial sums, then the inverse norm
    if (w) {
        w->x0 = reinterpret_cast<bf16*>(x0);
        w->x1 = reinterpret_cast<bf16*>(x1);
        w->a = reinterpret_cast<bf16*>(a);
        w->b = reinterpret_cast<bf16*>(b);
        w->part = reinterpret_cast<float*>(part);
    }
    return off;
}

int check_dims(int m, int n, int steps) {
    if (m < 8 || n < 8 || m % 8 != 0 || n % 8 != 0) return ZGCM_ERR_INVALID_ARG;
    if (steps < 0 || steps > 100) return ZGCM_ERR_INVALID_ARG;
    if ((long long)m * n >= (1LL << 40)) return ZGCM_ERR_UNSUPPORTED;
    return ZGCM_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The iterations from X0 (in w.x0, [p, q]); returns the buffer holding the result
cudaError_t iterate(Ws& w, int p, int q, int steps, float a, float b, float c, cudaStream_t stream, bf16** result) {
    bf16* x = w.x0;
    bf16* y = w.x1;
    cudaError_t e = cudaSuccess;
    for (int s = 0; s < steps && e == cudaSuccess; ++s) {
        // A = X X^T (symmetric: the upper tiles, then the mirror)
        if ((e = launch_gemm(x, x, nullptr, w.a, p, p, q, 1.0f, 0.0f, false, stream, true)) != cudaSuccess) break;
        if (c != 0.0f) {
            // B = b A + c A A  (A symmetric: A A = A A^T, and B symmetric)
            if ((e = launch_gemm(w.a, w.a, w.a, w.b, p, p, p, c, b, false, stream, true)) != cudaSuccess) break;
            // X' = a X + B X
            e = launch_gemm(w.b, x, x, y, p, q, p, 1.0f, a, true, stream);
        } else {
            // X' = a X + b (A X)
            e = launch_gemm(w.a, x, x, y, p, q, p, b, a, true, stream);
        }
        bf16* t = x;
        x = y;
        y = t;
    }
    *result = x;
    return e;
}

}  // namespace muon
}  // namespace zgcm

using namespace zgcm;
using namespace zgcm::muon;

extern "C" {

size_t zgcm_muon_workspace_size(int m, int n) {
    if (check_dims(m, n, 0) != ZGCM_OK) return 0;
    return ws_layout(m, n, nullptr, nullptr);
}

int zgcm_muon_gemm(const void* A, const void* B, const void* D, void* C, int M, int N, int K, float alpha,
                   float beta, int b_kn, void* cuda_stream) {
    if (M < 1 || N < 8 || K < 8 || N % 8 != 0 || K % 8 != 0) return ZGCM_ERR_INVALID_ARG;
    if (b_kn != 0 && b_kn != 1) return ZGCM_ERR_INVALID_ARG;
    if (!A || !B || !C) return ZGCM_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C) || (D && !aligned16(D))) return ZGCM_ERR_ALIGNMENT;
    const cudaError_t e = launch_gemm(static_cast<const bf16*>(A), static_cast<const bf16*>(B),
                                      static_cast<const bf16*>(D), static_cast<bf16*>(C), M, N, K, alpha,
                                      D ? beta : 0.0f, b_kn != 0, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}

int zgcm_muon_orthogonalize(const void* G, void* out, int m, int n, int steps, float a, float b, float c, float eps,
                            void* workspace, size_t workspace_bytes, void* cuda_stream) {
    int st = check_dims(m, n, steps);
    if (st != ZGCM_OK) return st;
    if (!G || !out) return ZGCM_ERR_INVALID_ARG;
    if (!aligned16(G) || !aligned16(out)) return ZGCM_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < zgcm_muon_workspace_size(m, n)) return ZGCM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ZGCM_ERR_ALIGNMENT;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    Ws w;
    ws_layout(m, n, static_cast<char*>(workspace), &w);
    const bool tall = m > n;
    const int p = tall ? n : m, q = tall ? m : n;
    const bf16* g = static_cast<const bf16*>(G);
    muon_sumsq_kernel<<<RED_BLOCKS, RED_THREADS, 0, stream>>>(g, (long long)m * n, w.part);
    muon_inv_norm_kernel<<<1, 32, 0, stream>>>(w.part, eps);
    const dim3 tb(32, 8), tg((n + 31) / 32, (m + 31) / 32);
    muon_scale_kernel<bf16><<<tg, tb, 0, stream>>>(g, w.x0, m, n, tall ? 1 : 0, w.part + RED_BLOCKS);
    cudaError_t e = cudaGetLastError();
    bf16* x = nullptr;
    if (e == cudaSuccess) e = iterate(w, p, q, steps, a, b, c, stream, &x);
    if (e == cudaSuccess) {
        // the result back in the caller's orientation ([p, q] -> [m, n])
        const dim3 og((q + 31) / 32, (p + 31) / 32);
        muon_scale_kernel<bf16><<<og, tb, 0, stream>>>(x, static_cast<bf16*>(out), p, q, tall ? 1 : 0, nullptr);
        e = cudaGetLastError();
    }
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}

int zgcm_muon_step(float* W, const void* G, float* M, int m, int n, float lr, float weight_decay, float momentum,
                   int steps, float a, float b, float c, float eps, void* workspace, size_t workspace_bytes,
                   void* cuda_stream) {
    int st = check_dims(m, n, steps);
    if (st != ZGCM_OK) return st;
    if (!W || !G || !M) return ZGCM_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(G) || !aligned16(M)) return ZGCM_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < zgcm_muon_workspace_size(m, n)) return ZGCM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ZGCM_ERR_ALIGNMENT;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    Ws w;
    ws_layout(m, n, static_cast<char*>(workspace), &w);
    const bool tall = m > n;
    const int p = tall ? n : m, q = tall ? m : n;
    muon_momentum_kernel<<<RED_BLOCKS, RED_THREADS, 0, stream>>>(M, static_cast<const bf16*>(G), (long long)m * n,
                                                                 momentum, w.part);
    muon_inv_norm_kernel<<<1, 32, 0, stream>>>(w.part, eps);
    const dim3 tb(32, 8), tg((n + 31) / 32, (m + 31) / 32);
    muon_scale_kernel<float><<<tg, tb, 0, stream>>>(M, w.x0, m, n, tall ? 1 : 0, w.part + RED_BLOCKS);
    cudaError_t e = cudaGetLastError();
    bf16* x = nullptr;
    if (e == cudaSuccess) e = iterate(w, p, q, steps, a, b, c, stream, &x);
    if (e == cudaSuccess) {
        muon_update_kernel<<<tg, tb, 0, stream>>>(W, x, m, n, tall ? 1 : 0, lr, weight_decay);
        e = cudaGetLastError();
    }
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}

}  // extern "C"
