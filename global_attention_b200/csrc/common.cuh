// common.cuh — device helpers shared by the gated window-attention kernels (sm_100a).
//
// Layer definition (what every kernel computes a part of):
//   QK-RMSNorm + partial RoPE + GQA 32/8 — shibing624 review of ZGCM-1, section "架构：5:1
//   的门控滑窗注意力"; window of the 128 nearest keys and full-causal global layers — ZGCM-1
//   summary (paper.rainbus.top), section "前置知识 / 滑动窗口注意力(SWA)与混合注意力";
//   sigmoid output gate — shibing624 review, section "架构" (formula lost; read as
//   out = sigmoid(g) * attn).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace zgcm {

constexpr int kD = 128;          // head dim (the only one supported)
constexpr int kMaxHalf = 64;     // max rope_dims / 2
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

typedef __nv_bfloat16 bf16;

// Everything a kernel needs, passed by value (__grid_constant__).
struct LayerParams {
    const bf16* q;       // [B,S,Hq,D]
    const bf16* k;       // [B,S,Hkv,D]
    const bf16* v;       // [B,S,Hkv,D]
    const bf16* g;       // [B,S,Hq,D]
    const float* gamma_q;
    const float* gamma_k;
    int B, S, Hq, Hkv, G;   // G = Hq / Hkv
    int rope_half;          // rope_dims / 2
    int W;                  // window (>= S means full causal)
    float eps;
    float scale;            // softmax scale
    float scale_log2;       // scale * log2(e)
    double theta[kMaxHalf]; // rope_base^(-2t/rope_dims), computed on the host in fp64
};

struct FwdParams {
    LayerParams L;
    bf16* out;    // [B,S,Hq,D]
    float* lse;   // [B,Hq,S]
};

// Activations the forward can leave for the backward (all null = none): the fp16 Q~
// [B,S,Hq,D] and K~ [B,S,Hkv,D] that both passes form, and the inverse RMS of every q and k
// row (fp32 [B,Hq,S], [B,Hkv,S]): the bits the backward's preparation would recompute.
struct SavedAct {
    void* q16 = nullptr;
    float* qrinv = nullptr;
    void* k16 = nullptr;
    float* krinv = nullptr;
};

struct BwdParams {
    LayerParams L;
    const bf16* out;    // [B,S,Hq,D]
    const float* lse;   // [B,Hq,S]
    const bf16* dout;   // [B,S,Hq,D]
    bf16* dq;           // [B,S,Hq,D]
    bf16* dk;           // [B,S,Hkv,D]
    bf16* dv;           // [B,S,Hkv,D]
    bf16* dg;           // [B,S,Hq,D]
    float* dgamma_q;    // [D]
    float* dgamma_k;    // [D]
    // workspace views
    float* delta;       // [B,Hq,S]   sum_j P_ij dP_ij (formed by the dq kernel)
    float* lse2;        // [B,Hq,S]   base-2 log-sum-exp of the backward's own scores
    bf16* dA;           // [B,S,Hq,D] dout * sigmoid(g), rounded to bf16 ("hi")
    bf16* dA_lo;        // [B,S,Hq,D] dout * sigmoid(g) - hi, rounded to bf16
    float* dgk_part;    // [n_k_parts, D]
    float* dgq_part;    // [n_q_parts, D]
    int n_k_parts, n_q_parts;
};

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ float bf2f(bf16 x) { return __bfloat162float(x); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// 1 / (1 + e^-x) with the fast reciprocal (2 ulp): an IEEE division here was a long
// instruction sequence per element of the streaming gate pass; for x < -88 the sum
// overflows and the quotient is 0.
__device__ __forceinline__ float sigmoidf_(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// cos/sin of the rotation angle pos * theta.  The product is formed and reduced modulo
// 2*pi in fp64 (the angle reaches ~2.6e5 rad at 256K positions, where an fp32 product
// would be off by ~0.016 rad), then the fp32 intrinsic evaluates the reduced angle.
__device__ __forceinline__ void rope_cs(double theta, int pos, float& c, float& s) {
    const double kTwoPi = 6.283185307179586;
    const double kInvTwoPi = 0.15915494309189535;
    double a = (double)pos * theta;
    double n = rint(a * kInvTwoPi);
    double r = fma(-n, kTwoPi, a);
    __sincosf((float)r, &s, &c);
}

// ---------------------------------------------------------------- row prologue
//
// One warp normalises and rotates one 128-wide row: lane l owns dims [4l, 4l+4).
//   r = sqrt(mean x^2 + eps); y = gamma * x / r;
//   pairs (t, t+half), t < half: y_t' = y_t c - y_{t+half} s ; y_{t+half}' = y_{t+half} c + y_t s
// `ybuf` is 128 floats of per-warp shared scratch.  Returns the rotated values in y[4]
// (xhat = x / r is formed first, then multiplied by gamma, as in the definition.)
__device__ __forceinline__ uint2 load_row4(const bf16* __restrict__ xrow) {
    return *reinterpret_cast<const uint2*>(xrow + 4 * (threadIdx.x & 31));
}

// `raw` holds this lane's 4 bf16 of the row (see load_row4).
__device__ __forceinline__ void prologue_row(uint2 raw, const float* gamma4, const LayerParams& L,
                                             int pos, float* ybuf, float y[4]) {
    const int lane = threadIdx.x & 31;
    float2 a = unpack_bf16(raw.x), b = unpack_bf16(raw.y);
    float x[4] = {a.x, a.y, b.x, b.y};
    float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
    ss = warp_sum(ss);
    float rinv = 1.0f / sqrtf(ss * (1.0f / kD) + L.eps);
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = (x[e] * rinv) * gamma4[e];
    const int half = L.rope_half;
    if (half > 0) {
        // lane t < half evaluates the angle of pair t once
        float ct = 1.f, st = 0.f;
        if (lane < half) rope_cs(L.theta[lane], pos, ct, st);
        // pairs t >= 32 (rope_dims > 64) are evaluated by the lane t - 32
        float ct2 = 1.f, st2 = 0.f;
        if (half > 32 && lane + 32 < half) rope_cs(L.theta[lane + 32], pos, ct2, st2);
        *reinterpret_cast<float4*>(ybuf + 4 * lane) = make_float4(y[0], y[1], y[2], y[3]);
        __syncwarp();
        float yn[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int d = 4 * lane + e;
            int t = d < half ? d : d - half;
            bool rot = d < 2 * half;
            int src = t & 31;
            float c0 = __shfl_sync(0xffffffffu, ct, src);
            float s0 = __shfl_sync(0xffffffffu, st, src);
            float c1 = __shfl_sync(0xffffffffu, ct2, src);
            float s1 = __shfl_sync(0xffffffffu, st2, src);
            float c = t < 32 ? c0 : c1, s = t < 32 ? s0 : s1;
            yn[e] = y[e];
            if (rot) {
                float partner = ybuf[d < half ? d + half : d - half];
                yn[e] = d < half ? y[e] * c - partner * s : y[e] * c + partner * s;
            }
        }
        __syncwarp();
#pragma unroll
        for (int e = 0; e < 4; ++e) y[e] = yn[e];
    }
}

// Backward of prologue_row for one row, warp-cooperative (lane l owns dims [4l, 4l+4)).
// dyrot[4]: gradient w.r.t. the rotated row.  Writes dx[4] (gradient w.r.t. raw x) and
// adds dy * xhat into dgamma_acc[4].
//   dy = R^T dyrot ; dxhat = dy * gamma ; dx = (dxhat - xhat * mean(dxhat * xhat)) / r
__device__ __forceinline__ void prologue_row_backward(uint2 raw, const float* gamma4,
                                                      const LayerParams& L, int pos, float* ybuf,
                                                      const float dyrot[4], float dx[4],
                                                      float dgamma_acc[4]) {
    const int lane = threadIdx.x & 31;
    float2 a = unpack_bf16(raw.x), b = unpack_bf16(raw.y);
    float x[4] = {a.x, a.y, b.x, b.y};
    float ss = warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    float r = sqrtf(ss * (1.0f / kD) + L.eps);
    float rinv = 1.0f / r;
    float dy[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) dy[e] = dyrot[e];
    const int half = L.rope_half;
    if (half > 0) {
        float ct = 1.f, st = 0.f, ct2 = 1.f, st2 = 0.f;
        if (lane < half) rope_cs(L.theta[lane], pos, ct, st);
        if (half > 32 && lane + 32 < half) rope_cs(L.theta[lane + 32], pos, ct2, st2);
        *reinterpret_cast<float4*>(ybuf + 4 * lane) = make_float4(dyrot[0], dyrot[1], dyrot[2], dyrot[3]);
        __syncwarp();
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int d = 4 * lane + e;
            int t = d < half ? d : d - half;
            bool rot = d < 2 * half;
            int src = t & 31;
            float c0 = __shfl_sync(0xffffffffu, ct, src);
            float s0 = __shfl_sync(0xffffffffu, st, src);
            float c1 = __shfl_sync(0xffffffffu, ct2, src);
            float s1 = __shfl_sync(0xffffffffu, st2, src);
            float c = t < 32 ? c0 : c1, s = t < 32 ? s0 : s1;
            if (rot) {
                float partner = ybuf[d < half ? d + half : d - half];
                // d <  half: dy_t      =  dyrot_t c + dyrot_{t+half} s
                // d >= half: dy_{t+h}  = -dyrot_t s + dyrot_{t+half} c
                dy[e] = d < half ? dyrot[e] * c + partner * s : dyrot[e] * c - partner * s;
            }
        }
        __syncwarp();
    }
    float xhat[4], dxh[4];
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        xhat[e] = x[e] * rinv;
        dxh[e] = dy[e] * gamma4[e];
        m += dxh[e] * xhat[e];
        dgamma_acc[e] += dy[e] * xhat[e];
    }
    m = warp_sum(m) * (1.0f / kD);
#pragma unroll
    for (int e = 0; e < 4; ++e) dx[e] = (dxh[e] - xhat[e] * m) * rinv;
}

// ---------------------------------------------------------------- tensor-core (mma.sync) helpers

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// D(16x8 fp32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Row-major [rows][128] bf16 tile in shared memory, 256 B per row, with the 16-byte chunk
// index XOR-swizzled by (row & 7) so that 8 consecutive rows of one chunk column hit 8
// different bank groups (ldmatrix reads conflict-free).
__device__ __forceinline__ uint32_t tile_off(int row, int chunk) {
    return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* gptr, bool pred) {
    int n = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(gptr), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

}  // namespace zgcm
