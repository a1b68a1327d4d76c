// bwd_tc.cuh — pieces shared by the tcgen05 backward kernels (sm_100a): the parameter block,
// the layout of the per-row arrays, power-of-two fitting for fp16 operands, and the
// one-thread-per-row RoPE / RMSNorm backward of the dq and dk epilogues.  Definitions of the
// layer and page citations: common.cuh.
#pragma once
#include <cudaTypedefs.h>

#include "tc_rows.cuh"

namespace zgcm {
using namespace sm100;

constexpr int TB_THREADS = 512;
constexpr int TB_MAX_GRID = 1024;  // partial-sum slots reserved in the workspace

struct BwdTcParams {
    CUtensorMap tm_q;   // {D, Hq, S, B}, box {64, 1, 128, 1}, 128B swizzle
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    CUtensorMap tm_da;  // dA16, fp16, same geometry as tm_q
    CUtensorMap tm_k16; // K~ fp16 (normalised, rotated, times the q~/k~ scale), geometry of tm_k
    CUtensorMap tm_v16; // V fp16 times 2^e per 128-row tile, geometry of tm_v
    CUtensorMap tm_q16; // Q~ fp16 (normalised, rotated, times the q~/k~ scale), geometry of tm_q
    CUtensorMap tm_q16h;  // the same with 64-row boxes (key-major kernel, one 64-query half)
    CUtensorMap tm_dah;   // dA16 with 64-row boxes
    CUtensorMap tm_lse;   // lse2p, Delta, 2^-e of the dA rows: fp32 {Spad, Hq, B}, box {64, 1, 1}
    CUtensorMap tm_delta;
    CUtensorMap tm_dainv;
    BwdParams P;
    const __half* da16; // [B,S,Hq,D] dA * 2^e (e per row)
    float* dainv;       // [B,Hq,Spad] 2^-e of each dA row (0 for an all-zero row and past S)
    float* domax;       // [B,Hq,Spad] max |dout| of each row (bound on |dA|)
    float* krinv;       // [B,Hkv,S] inverse RMS of each raw k row
    float* qrinv;       // [B,Hq,S] inverse RMS of each raw q row
    float* lse2p;       // [B,Hq,Spad] the forward's lse in base 2 (+inf past S), for TMA
    float* vnorm;       // [B,Hkv,S] 2-norm of each raw v row
    float* vtinv;       // [B,Hkv,ceil(S/128)] 2^-e of each V tile
    float* tstat;       // [3][B,Hkv,ceil(S/128)] per-tile max |dout|, max |Delta|, max ||v||
                        // (wide windows only; null for the sliding-window kernels)
    int* err;
    int total;          // steps (query-major) or units (key-major)
    int wide;           // 1: window wider than one tile (key-major: heaviest unit first, one
                        // unit per CTA, unit scales from tstat)
};

// Row stride of the backward's per-row arrays [B, Hq, Spad]: the sequence rounded up to 64,
// so that a 64-row run starts on a 256-byte boundary and the arrays can be TMA tensors (a
// global stride must be a multiple of 16 bytes).  Entries past S hold neutral values.
__host__ __device__ __forceinline__ int row_stride(int S) { return (S + 63) & ~63; }

// First key tile a query row sees in a wide-window problem whose query rows start at q_off
// (window W <= S): the tile of key q_off - W + 1; 0 when that is before the sequence.
__host__ __device__ __forceinline__ int wide_first_tile(const LayerParams& L) {
    const int j = L.q_off - L.W + 1;
    return j > 0 ? j / TF_BN : 0;
}

// power-of-two exponent e with |x| * 2^e in [2^13, 2^14); 0 for x == 0 or non-finite
__device__ __forceinline__ int fit_exp(float x) {
    if (!(x > 0.f) || !isfinite(x)) return 0;
    int e = 13 - ilogbf(x);
    return max(-120, min(120, e));
}

// 32 lanes x 16 consecutive 32-bit columns load
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Sum of v[e] over the 32 lanes of the warp for e = 0..31, delivered as: lane L returns the
// total of index L (recursive halving; 31 shuffles).  v is clobbered.
__device__ __forceinline__ float warp_transpose_sum(float* v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
        const bool upper = (lane & k) != 0;
#pragma unroll
        for (int j = 0; j < k; ++j) {
            const float send = upper ? v[j] : v[j + k];
            const float keep = upper ? v[j + k] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, k);
        }
    }
    return v[0];
}

// swizzled 16-byte chunk ch (0..15, 8 values each) of row r in a two-half 128-row tile
__device__ __forceinline__ uint4* tile_chunk(unsigned char* h0, unsigned char* h1, int r, int ch) {
    unsigned char* hb = ch < 8 ? h0 : h1;
    return reinterpret_cast<uint4*>(hb + (uint32_t)r * 128u + (uint32_t)(((ch & 7) ^ (r & 7)) << 4));
}

// RoPE / RMSNorm backward of one row held by one thread, one pass over the row:
//   dy = R^T (f * dq~)       (dq~: the row's 128 accumulator columns, copied out of TMEM
//                             into registers so that the tensor memory is released first;
//                             R rotates pairs (t, t+21) at `pos`)
//   dx = (dy * gamma - xhat * mdot) * rinv,   xhat = x * rinv,   d_gamma += dy * xhat
// The caller supplies rinv = 1/sqrt(mean x^2 + eps) (from the prologue) and
// mdot = mean_d(dy_d gamma_d xhat_d).  Because R is orthogonal and q~ = R(gamma * xhat),
// mdot = (q~ . dq~) / D, which the softmax warps form as a row sum of dS * S; so the raw row
// x (global memory) is read once: its first 64 values prefetched by the caller (xv0), the
// last 64 here.  d_gamma goes into this warp's slice `dgam` through warp-transposed sums
// (lane L owns one dimension per 32-wide block: a fixed summation order, reproducible).
// `valid` masks rows past the sequence (they still join the collectives).
// cs_at(t): (cos, sin) of pair t at the row's position (rope_cs), so that a caller with
// several heads of one row can form them once.
// RH: the number of rotated pairs when known at compile time (the layer's 21, unrolled), or 0
// for any number rh (0..64) given at run time.
template <int RH = TF_HALF, class CsAt>
__device__ __forceinline__ void row_rope_rms_backward_cs(float (&dy)[128], float f, float mdot, float rinv,
                                                         const uint4 (&xv0)[8], const bf16* x, bf16* dst,
                                                         bool valid, CsAt cs_at, const float* gamma, float* dgam,
                                                         int rh = RH) {
    const int lane = threadIdx.x & 31;
    const uint4* xr = reinterpret_cast<const uint4*>(x);
    uint4* dr = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int e = 0; e < 128; ++e) dy[e] *= f;
    // transpose of the rotation of pairs (t, t + rh)
    if constexpr (RH > 0) {
#pragma unroll
        for (int t = 0; t < RH; ++t) {
            const float2 w = cs_at(t);
            const float c = w.x, s = w.y;
            const float d1 = dy[t], d2 = dy[t + RH];
            dy[t] = d1 * c + d2 * s;
            dy[t + RH] = d2 * c - d1 * s;
        }
    } else {
#pragma unroll 1
        for (int t = 0; t < rh; ++t) {
            const float2 w = cs_at(t);
            const float c = w.x, s = w.y;
            const float d1 = dy[t], d2 = dy[t + rh];
            dy[t] = d1 * c + d2 * s;
            dy[t + rh] = d2 * c - d1 * s;
        }
    }
    uint4 xv1[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) xv1[c] = valid ? __ldg(xr + 8 + c) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // dims [32 q, 32 q + 32)
        float* v = dy + 32 * q;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 u = q < 2 ? xv0[4 * q + c] : xv1[4 * (q - 2) + c];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 t = unpack_bf16(w[e]);
                const int d = 8 * c + 2 * e, gd = 32 * q + d;
                const float x0 = t.x * rinv, x1 = t.y * rinv;
                o[e] = pack_bf16((v[d] * gamma[gd] - x0 * mdot) * rinv, (v[d + 1] * gamma[gd + 1] - x1 * mdot) * rinv);
                v[d] *= x0;
                v[d + 1] *= x1;
            }
            if (valid) dr[4 * q + c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        const float tot = warp_transpose_sum(v);
        dgam[32 * q + lane] += tot;
    }
}

template <int RH = TF_HALF>
__device__ __forceinline__ void row_rope_rms_backward_regs(float (&dy)[128], float f, float mdot, float rinv,
                                                           const uint4 (&xv0)[8], const bf16* x, bf16* dst,
                                                           bool valid, int pos, const float* gamma, float* dgam,
                                                           const LayerParams& L) {
    row_rope_rms_backward_cs<RH>(dy, f, mdot, rinv, xv0, x, dst, valid,
                                 [&](int t) {
                                     float c, s;
                                     rope_cs(L.theta[t], pos, c, s);
                                     return make_float2(c, s);
                                 },
                                 gamma, dgam, L.rope_half);
}


// Kernels of the wide-window / global backward (bwd_glob_sm100.cu), launched with the
// sliding-window ones by launch_bwd_tc.
__global__ void bwd_tile_stats_kernel(const __grid_constant__ BwdTcParams p);
// the wide query-major kernel, its instance for the number of rotated pairs
cudaError_t launch_bwd_q_glob(const BwdTcParams& p, int units, cudaStream_t stream);

constexpr int BQG_THREADS = 384;
constexpr int BTS_THREADS = 128;

}  // namespace zgcm
