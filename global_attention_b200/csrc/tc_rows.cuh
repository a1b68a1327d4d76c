// tc_rows.cuh — row-per-thread pieces shared by the tcgen05 kernels (sm_100a): the
// sweep's step decoding, fast MUFU exp2/tanh, rotation angles, and the in-place
// RMSNorm + partial-RoPE prologue of a swizzled 128-row tile.  Definitions of the layer
// and page citations: common.cuh.
#pragma once
#include <cuda_fp16.h>

#include "sm100.cuh"

namespace zgcm {

constexpr int TF_BM = 128;
constexpr int TF_BN = 128;
constexpr int TF_HALF = 21;              // rotated pairs (rope_dims = 42)
constexpr uint32_t TF_TILE_BYTES = TF_BN * kD * 2;   // one 128 x 128 16-bit tile
constexpr uint32_t TF_HALF_BYTES = TF_BN * 64 * 2;   // one 128-row x 64-col half: 16 KB
constexpr uint32_t TF_RING_HALF = 2 * TF_HALF_BYTES; // one d-half of a 2-slot ring: 32 KB

struct StepInfo {
    int b, kvh, qb;
    bool fresh;        // first step of a chain in this CTA: load the previous tile too
    bool release_cur;  // the next step does not reuse this step's current tile
};

__device__ __forceinline__ StepInfo decode_step(const LayerParams& L, int t, int t_begin, int t_end) {
    const int nqb = (L.S + TF_BM - 1) / TF_BM;
    StepInfo s;
    const int chain = t / nqb;
    s.qb = t - chain * nqb;
    s.b = chain / L.Hkv;
    s.kvh = chain - s.b * L.Hkv;
    s.fresh = (t == t_begin) || (s.qb == 0);
    s.release_cur = (t + 1 >= t_end) || (s.qb + 1 == nqb);
    return s;
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float fast_tanh(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Power of two that keeps the fp16 q~, k~ in range: |y_d| <= sqrt(D) max|gamma|.  Every CTA
// of the forward and of both backward kernels derives the same value from gamma_q, gamma_k
// in shared memory, so all of them form bit-identical fp16 q~, k~ and scores.
__device__ __forceinline__ float qk_fp16_scale(const float* gq, const float* gk) {
    float gmax = 0.f;
    for (int d = 0; d < kD; ++d) gmax = fmaxf(gmax, fmaxf(fabsf(gq[d]), fabsf(gk[d])));
    const float bound = gmax * sqrtf((float)kD);
    return (bound > 16384.f && isfinite(bound)) ? ldexpf(1.0f, 13 - ilogbf(bound)) : 1.0f;
}

// Bits lo..hi of a 32-bit word, clamped to 0..31 (0 when the range is empty): the visible
// positions of a 32-wide chunk for one thread's row.  A bit test and a select per element
// replace the window comparisons, which compiled to divergent branches around the exp2.
__device__ __forceinline__ uint32_t bit_range(int lo, int hi) {
    lo = max(lo, 0);
    hi = min(hi, 31);
    if (lo > hi) return 0u;
    return (0xffffffffu >> (31 - hi)) & (0xffffffffu << lo);
}

// ------------------------------------------------------------------ prologue (one row per thread)

// cos/sin of the TF_HALF rotation angles at `pos`, into column r of the table
__device__ __forceinline__ void tf_angles(const LayerParams& L, int pos, float2 (*cs)[TF_BM], int r) {
#pragma unroll 1  // rolled: unrolled, the fp64 angle products of all 21 pairs stay live and spill
    for (int t = 0; t < TF_HALF; ++t) {
        float c, s;
        rope_cs(L.theta[t], pos, c, s);
        cs[t][r] = make_float2(c, s);
    }
}

// Row `r` of a 128-row tile stored as two 16 KB d-halves (h0, h1), 128-byte swizzled:
// normalise (RMS, gamma), rotate pairs (t, t+21) for t < 21, multiply by `oscale` (a power
// of two, 1 unless the fp16 range needs it) and write back in place as bf16 (F16 = false)
// or fp16.  Rows outside the sequence are zero-filled by TMA and stay zero.  Returns the
// row's inverse RMS (the backward's epilogue reuses it).
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    if constexpr (F16) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    } else {
        return pack_bf16(a, b);
    }
}

// cs_at(t) gives (cos, sin) of pair t at the row's position: from the shared table
// (tf_prologue_row) or from registers (the preparation kernel).  Same values, same bits.
template <bool F16, class CsAt>
__device__ __forceinline__ float tf_prologue_row_at(unsigned char* h0, unsigned char* h1, int r, const float* gamma,
                                                   const LayerParams& L, CsAt cs_at, float oscale) {
    // chunk ch (8 dims, 16 bytes) of the row: half ch / 8, swizzled position (ch % 8) ^ (r % 8)
    auto chunk = [&](int ch) -> uint4* {
        unsigned char* hb = ch < 8 ? h0 : h1;
        return reinterpret_cast<uint4*>(hb + (uint32_t)r * 128u + (uint32_t)(((ch & 7) ^ (r & 7)) << 4));
    };
    float ss = 0.f;
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {
        const uint4 u = *chunk(ch);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = unpack_bf16(w[e]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
        }
    }
    // a zero row (outside the sequence, zero-filled by TMA) stays zero even with eps = 0
    const float rinv1 = ss > 0.f ? rsqrtf(fmaf(ss, 1.0f / kD, L.eps)) : 0.f;
    const float rinv = rinv1 * oscale;
    // dims 0..47 (chunks 0..5): normalise, rotate the first 42
    float y[48];
#pragma unroll
    for (int ch = 0; ch < 6; ++ch) {
        const uint4 u = *chunk(ch);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = unpack_bf16(w[e]);
            const int d = ch * 8 + 2 * e;
            y[d] = (f.x * rinv) * gamma[d];
            y[d + 1] = (f.y * rinv) * gamma[d + 1];
        }
    }
    // explicit fused multiply-adds (here and in the mean square above): every kernel that forms
    // q~ or k~ (the forwards, the backward's preparation, the strip kernels' in-place
    // conversion) rounds identically, whatever contraction the compiler would pick at each site
#pragma unroll
    for (int t = 0; t < TF_HALF; ++t) {
        const float a = y[t], bb = y[t + TF_HALF];
        const float2 w = cs_at(t);
        y[t] = fmaf(a, w.x, -(bb * w.y));
        y[t + TF_HALF] = fmaf(bb, w.x, a * w.y);
    }
#pragma unroll
    for (int ch = 0; ch < 6; ++ch) {
        uint4 o;
        o.x = pack2<F16>(y[ch * 8 + 0], y[ch * 8 + 1]);
        o.y = pack2<F16>(y[ch * 8 + 2], y[ch * 8 + 3]);
        o.z = pack2<F16>(y[ch * 8 + 4], y[ch * 8 + 5]);
        o.w = pack2<F16>(y[ch * 8 + 6], y[ch * 8 + 7]);
        *chunk(ch) = o;
    }
    // dims 48..127: normalise only
#pragma unroll
    for (int ch = 6; ch < 16; ++ch) {
        const uint4 u = *chunk(ch);
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = unpack_bf16(w[e]);
            const int d = ch * 8 + 2 * e;
            w[e] = pack2<F16>((f.x * rinv) * gamma[d], (f.y * rinv) * gamma[d + 1]);
        }
        *chunk(ch) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return rinv1;  // 1 / sqrt(mean x^2 + eps) of the row (0 for a zero row)
}

// Element d (0..127) of row r in a two-half 128-row tile with 128-byte swizzle: its address.
__device__ __forceinline__ unsigned char* tile_elem(unsigned char* h0, unsigned char* h1, int r, int d) {
    unsigned char* hb = d < 64 ? h0 : h1;
    const int dd = d & 63;
    return hb + (uint32_t)r * 128u + (uint32_t)(((((dd >> 3) ^ (r & 7)) << 4)) + ((dd & 7) << 1));
}

// The same normalisation and rotation as tf_prologue_row_at for any number of rotated pairs
// L.rope_half (0..64, pairs (t, t + rope_half)), the angles formed at `pos` as needed: each
// pair's two elements are read, rotated and written back in place.  The arithmetic and its
// rounding are those of tf_prologue_row_at, so for 21 pairs both give the same bits.
template <bool F16>
__device__ __forceinline__ float tf_prologue_row_any(unsigned char* h0, unsigned char* h1, int r, const float* gamma,
                                                    const LayerParams& L, int pos, float oscale) {
    float ss = 0.f;
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {
        const uint4 u = *reinterpret_cast<const uint4*>(tile_elem(h0, h1, r, 8 * ch));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = unpack_bf16(w[e]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
        }
    }
    const float rinv1 = ss > 0.f ? rsqrtf(fmaf(ss, 1.0f / kD, L.eps)) : 0.f;
    const float rinv = rinv1 * oscale;
    auto ld = [&](int d) { return __bfloat162float(*reinterpret_cast<const bf16*>(tile_elem(h0, h1, r, d))); };
    auto st = [&](int d, float v) {
        if constexpr (F16)
            *reinterpret_cast<__half*>(tile_elem(h0, h1, r, d)) = __float2half_rn(v);
        else
            *reinterpret_cast<bf16*>(tile_elem(h0, h1, r, d)) = __float2bfloat16_rn(v);
    };
    const int rh = L.rope_half;
#pragma unroll 1
    for (int t = 0; t < rh; ++t) {
        const float a = (ld(t) * rinv) * gamma[t], bb = (ld(t + rh) * rinv) * gamma[t + rh];
        float c, sn;
        rope_cs(L.theta[t], pos, c, sn);
        st(t, fmaf(a, c, -(bb * sn)));
        st(t + rh, fmaf(bb, c, a * sn));
    }
#pragma unroll 1
    for (int d = 2 * rh; d < kD; ++d) st(d, (ld(d) * rinv) * gamma[d]);
    return rinv1;
}

template <bool F16 = false>
__device__ __forceinline__ float tf_prologue_row(unsigned char* h0, unsigned char* h1, int r, const float* gamma,
                                                const LayerParams& L, const float2 (*cs)[TF_BM],
                                                float oscale = 1.0f) {
    return tf_prologue_row_at<F16>(h0, h1, r, gamma, L, [&](int t) { return cs[t][r]; }, oscale);
}


}  // namespace zgcm
