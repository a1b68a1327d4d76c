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
    const bf16* q;       // [B,Sq,Hq,D]: the query rows, positions q_off .. S-1
    const bf16* k;       // [B,S,Hkv,D]
    const bf16* v;       // [B,S,Hkv,D]
    const bf16* g;       // [B,Sq,Hq,D]
    const float* gamma_q;
    const float* gamma_k;
    int B, S, Hq, Hkv, G;   // G = Hq / Hkv
    int rope_half;          // rope_dims / 2
    int W;                  // window (>= S means full causal)
    int q_off;              // position of the first query row (0: every position has one;
                            // else a multiple of 128, wide windows only).  q, g, out, lse,
                            // dout, dq, dg hold rows q_off .. S-1; k, v, dk, dv all S rows.
    int Sq;                 // S - q_off
    float eps;
    float scale;            // softmax scale
    float scale_log2;       // scale * log2(e)
    double theta[kMaxHalf]; // rope_base^(-2t/rope_dims), computed on the host in fp64
};

struct FwdParams {
    LayerParams L;
    bf16* out;    // [B,Sq,Hq,D]
    float* lse;   // [B,Hq,Sq]
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
    const bf16* out;    // [B,Sq,Hq,D]
    const float* lse;   // [B,Hq,Sq]
    const bf16* dout;   // [B,Sq,Hq,D]
    bf16* dq;           // [B,Sq,Hq,D]
    bf16* dk;           // [B,S,Hkv,D]
    bf16* dv;           // [B,S,Hkv,D]
    bf16* dg;           // [B,Sq,Hq,D]
    float* dgamma_q;    // [D]
    float* dgamma_k;    // [D]
    // workspace views (set by the launcher)
    float* delta;       // [B,Hq,Spad] Delta of each row
    float* dgk_part;    // [slots, D] d_gamma_k partial sums
    float* dgq_part;    // [slots, D] d_gamma_q partial sums
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


}  // namespace zgcm
