// decode.cu — one decode step of the gated attention layer: a single new token per sequence
// against a KV cache (the inference path of the 27 sliding layers, whose cache is a ring of
// W slots, and of the global layers, whose cache grows; the ZGCM-1 KV-cache design: pages
// cited in include/zgcm_attn.h and common.cuh).
//
// For sequence b at position p = pos[b]:
//   q~ = RoPE(gamma_q * q / rms(q)), k~ = RoPE(gamma_k * k / rms(k)) at position p;
//   the cache slot p mod C receives k~ (fp16, times the power-of-two scale qk_fp16_scale of
//   the training kernels, so the cached keys are the training forward's K~ values) and v;
//   out = sigmoid(g) * softmax_{j in [p-W+1, p]}(scale q~.k~_j) v_j,   lse as in the forward.
//
// Decode is bound by reading the cache (each step reads every visible key and value once),
// so it runs on CUDA cores with coalesced 8-byte loads, not on the tensor cores (the 4 query
// heads of a KV group are far too few rows for a 128-row MMA tile).  Two kernels:
//   decode_split_kernel    CTA = (b, KV head, split of the visible keys); warp = query head
//                          of the group; lane = 4 head dims.  Online softmax over the split's
//                          keys; partial (max, sum, O) to the workspace.  The CTA whose split
//                          holds position p also normalises k, writes the cache slot and uses
//                          the cached (fp16) value like every other key.
//   decode_combine_kernel  CTA = (b, query head), thread = head dim: merges the splits,
//                          applies the gate, writes out and lse.
#include "bwd_tc.cuh"  // warp_transpose_sum

namespace zgcm {

constexpr int DEC_THREADS = 128;        // 4 warps
constexpr int DEC_WARPS = DEC_THREADS / 32;
constexpr int DEC_KEYS = 512;           // keys per split (CTA)
constexpr int DEC_KB = 8;               // keys per batch
constexpr int DEC_GH = 4;               // query heads per pass: DEC_GH x DEC_KB = 32 scores, one per lane
constexpr int DEC_REC = 4 + kD;         // floats per partial record: max, sum, 2 pad, O (16-byte aligned)

struct DecodeParams {
    LayerParams L;          // q, k, v, g: the new token ([B,Hq,D] / [B,Hkv,D]); S unused
    const int* pos;         // [B] position of the new token
    __half* kc;             // [B,C,Hkv,D] K~ * oscale, fp16
    bf16* vc;               // [B,C,Hkv,D]
    int C;                  // cache slots per sequence
    int nsplit;             // splits of the visible keys (ceil(min(W, C) / DEC_KEYS))
    float* part;            // [B*Hq][nsplit * DEC_WARPS][DEC_REC]: max (base 2), sum, pad, O (relative to max)
    bf16* out;              // [B,Hq,D]
    float* lse;             // [B,Hq]
};

// CTA = (b, KV head, split of DEC_KEYS visible keys).  The split's keys go to the 4 warps in
// batches of 8 (batch i to warp i mod 4); a warp takes all the group's query heads (4 per
// pass), so every cached row is loaded once per CTA.  Per batch, lane l holds the partial dot
// products of its 4 head dims for the 4 x 8 (head, key) pairs; one transposed warp sum (31
// shuffles) leaves the score of pair l = (head l/8, key l%8) in lane l; the heads' max and
// sum run over their 8 lanes; the O update takes each pair's weight from its lane.  Each
// warp writes its own partial record (max, sum, O) per head.
__global__ void __launch_bounds__(DEC_THREADS) decode_split_kernel(const __grid_constant__ DecodeParams p) {
    const LayerParams& L = p.L;
    __shared__ __align__(16) float gq[kD];
    __shared__ __align__(16) float gk[kD];
    __shared__ __align__(16) float ybuf[DEC_WARPS][kD];  // prologue_row's per-warp scratch (float4 stores)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x / L.Hkv, kvh = blockIdx.x % L.Hkv, s = blockIdx.y;
    gq[tid] = L.gamma_q[tid];
    gk[tid] = L.gamma_k[tid];
    __syncthreads();
    const float oscale = qk_fp16_scale(gq, gk);  // the training kernels' K~ scale
    const int pos = p.pos[b];
    const int lo = max(0, pos - L.W + 1);
    const int j0 = lo + s * DEC_KEYS, j1 = min(pos + 1, j0 + DEC_KEYS);   // this split's keys
    // the visible keys must all still be in the cache (a ring of C slots)
    const bool fits = pos >= 0 && pos - lo + 1 <= p.C;
    const size_t kv_row = (size_t)L.Hkv * kD;  // elements between consecutive cache slots

    // the new key and value into slot pos mod C (the split that holds position pos)
    if (fits && pos >= j0 && pos < j1 && warp < 2) {
        const size_t slot = ((size_t)b * p.C + pos % p.C) * kv_row + (size_t)kvh * kD + 4 * lane;
        const size_t src = ((size_t)b * L.Hkv + kvh) * kD;
        if (warp == 0) {
            float y[4];
            prologue_row(load_row4(L.k + src), gk + 4 * lane, L, pos, ybuf[0], y);
            __half2 h01 = __floats2half2_rn(y[0] * oscale, y[1] * oscale);
            __half2 h23 = __floats2half2_rn(y[2] * oscale, y[3] * oscale);
            uint2 w;
            w.x = *reinterpret_cast<uint32_t*>(&h01);
            w.y = *reinterpret_cast<uint32_t*>(&h23);
            *reinterpret_cast<uint2*>(p.kc + slot) = w;
        } else {
            *reinterpret_cast<uint2*>(p.vc + slot) = *reinterpret_cast<const uint2*>(L.v + src + 4 * lane);
        }
    }
    __syncthreads();  // the new cache entry is read below like every other key

    const float c2 = L.scale_log2 / oscale;  // q~ (fp32) . (k~ oscale) -> base-2 score
    const int nb = j1 > j0 ? (j1 - j0 + DEC_KB - 1) / DEC_KB : 0;
    const int hl = lane >> 3, kl = lane & 7;      // the (head, key) pair of this lane's score
    const size_t head_off = (size_t)kvh * kD + 4 * lane;
    for (int hg0 = 0; hg0 < L.G; hg0 += DEC_GH) {
        const int nh = min(DEC_GH, L.G - hg0);
        float q[DEC_GH][4];
#pragma unroll
        for (int h = 0; h < DEC_GH; ++h) {
            if (h < nh) {
                prologue_row(load_row4(L.q + ((size_t)b * L.Hq + kvh * L.G + hg0 + h) * kD), gq + 4 * lane, L, pos,
                             ybuf[warp], q[h]);
            } else {
                q[h][0] = q[h][1] = q[h][2] = q[h][3] = 0.f;
            }
        }
        float m[DEC_GH], l[DEC_GH], o[DEC_GH][4];
#pragma unroll
        for (int h = 0; h < DEC_GH; ++h) {
            m[h] = fits ? -INFINITY : NAN;   // a window longer than the cache: no valid answer
            l[h] = fits ? 0.f : NAN;
            o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
        }
        for (int bi = warp; fits && bi < nb; bi += DEC_WARPS) {
            const int jb = j0 + bi * DEC_KB, nk = min(DEC_KB, j1 - jb);
            uint2 kw[DEC_KB], vw[DEC_KB];
#pragma unroll
            for (int t = 0; t < DEC_KB; ++t) {  // keys past the split's end load its last key (masked)
                const size_t off = ((size_t)b * p.C + (jb + min(t, nk - 1)) % p.C) * kv_row + head_off;
                kw[t] = *reinterpret_cast<const uint2*>(p.kc + off);
                vw[t] = *reinterpret_cast<const uint2*>(p.vc + off);
            }
            float v[DEC_GH * DEC_KB];  // partial dots, index h * DEC_KB + key
#pragma unroll
            for (int t = 0; t < DEC_KB; ++t) {
                const float2 k01 = __half22float2(*reinterpret_cast<const __half2*>(&kw[t].x));
                const float2 k23 = __half22float2(*reinterpret_cast<const __half2*>(&kw[t].y));
#pragma unroll
                for (int h = 0; h < DEC_GH; ++h)
                    v[h * DEC_KB + t] = q[h][0] * k01.x + q[h][1] * k01.y + q[h][2] * k23.x + q[h][3] * k23.y;
            }
            const float tot = warp_transpose_sum(v);
            const float sc = (kl < nk && hl < nh) ? tot * c2 : -INFINITY;
            // each head's batch maximum over its 8 lanes, then every lane learns all four
            float gm = sc;
            gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, 4));
            gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, 2));
            gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, 1));
            float mn[DEC_GH];
#pragma unroll
            for (int h = 0; h < DEC_GH; ++h) {
                mn[h] = fmaxf(m[h], __shfl_sync(0xffffffffu, gm, 8 * h));
                if (mn[h] > m[h]) {   // the same decision on every lane
                    const float a = fast_exp2(m[h] - mn[h]);  // 0 from the empty start
                    l[h] *= a;
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[h][e] *= a;
                    m[h] = mn[h];
                }
            }
            const float mh = hl == 0 ? mn[0] : hl == 1 ? mn[1] : hl == 2 ? mn[2] : mn[3];
            const float pl = sc == -INFINITY ? 0.f : fast_exp2(sc - mh);
            float gs = pl;
            gs += __shfl_xor_sync(0xffffffffu, gs, 4);
            gs += __shfl_xor_sync(0xffffffffu, gs, 2);
            gs += __shfl_xor_sync(0xffffffffu, gs, 1);
#pragma unroll
            for (int h = 0; h < DEC_GH; ++h) l[h] += __shfl_sync(0xffffffffu, gs, 8 * h);
#pragma unroll
            for (int t = 0; t < DEC_KB; ++t) {
                const float2 v01 = unpack_bf16(vw[t].x), v23 = unpack_bf16(vw[t].y);
#pragma unroll
                for (int h = 0; h < DEC_GH; ++h) {
                    const float ph = __shfl_sync(0xffffffffu, pl, 8 * h + t);
                    o[h][0] = fmaf(ph, v01.x, o[h][0]);
                    o[h][1] = fmaf(ph, v01.y, o[h][1]);
                    o[h][2] = fmaf(ph, v23.x, o[h][2]);
                    o[h][3] = fmaf(ph, v23.y, o[h][3]);
                }
            }
        }
        const int nrec = p.nsplit * DEC_WARPS;
#pragma unroll
        for (int h = 0; h < DEC_GH; ++h) {
            if (h >= nh) break;
            const int hq = kvh * L.G + hg0 + h;
            float* part = p.part + (((size_t)b * L.Hq + hq) * nrec + s * DEC_WARPS + warp) * DEC_REC;
            if (lane == 0) *reinterpret_cast<float4*>(part) = make_float4(m[h], l[h], 0.f, 0.f);
            *reinterpret_cast<float4*>(part + 4 + 4 * lane) = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
        }
    }
}

__global__ void __launch_bounds__(kD) decode_combine_kernel(const __grid_constant__ DecodeParams p) {
    const LayerParams& L = p.L;
    const int d = threadIdx.x, bh = blockIdx.x;
    const int nrec = p.nsplit * DEC_WARPS;
    const float* part = p.part + (size_t)bh * nrec * DEC_REC;
    float m = -INFINITY;
    bool bad = false;  // a split marked the window as longer than the cache
    for (int s = 0; s < nrec; ++s) {
        const float ms = part[s * DEC_REC];
        bad |= isnan(ms);
        m = fmaxf(m, ms);
    }
    float l = 0.f, o = 0.f;
    for (int s = 0; s < nrec; ++s) {
        const float* ps = part + s * DEC_REC;
        if (ps[0] == -INFINITY) continue;   // a split past the last key: empty
        const float a = exp2f(ps[0] - m);
        l = fmaf(ps[1], a, l);
        o = fmaf(ps[4 + d], a, o);
    }
    if (bad) l = o = NAN;
    const float gx = __bfloat162float(L.g[(size_t)bh * kD + d]);
    const float sg = 1.0f / (1.0f + expf(-gx));
    p.out[(size_t)bh * kD + d] = __float2bfloat16_rn(sg * (o / l));
    if (d == 0) p.lse[bh] = (m + log2f(l)) * kLn2;
}

size_t decode_workspace_bytes(int B, int Hq, int window, int C) {
    const int vis = window < C ? window : C;
    const size_t nsplit = (size_t)((vis + DEC_KEYS - 1) / DEC_KEYS);
    return (size_t)B * Hq * nsplit * DEC_WARPS * DEC_REC * sizeof(float);
}

cudaError_t launch_decode(const LayerParams& L, const int* pos, void* k_cache, void* v_cache, int C, void* out,
                          float* lse, void* workspace, cudaStream_t stream) {
    DecodeParams p;
    p.L = L;
    p.pos = pos;
    p.kc = static_cast<__half*>(k_cache);
    p.vc = static_cast<bf16*>(v_cache);
    p.C = C;
    const int vis = L.W < C ? L.W : C;
    p.nsplit = (vis + DEC_KEYS - 1) / DEC_KEYS;
    p.part = static_cast<float*>(workspace);
    p.out = static_cast<bf16*>(out);
    p.lse = lse;
    const long long ctas = (long long)L.B * L.Hkv;
    if (ctas > 0x7fffffffLL || p.nsplit > 65535 || (long long)L.B * L.Hq > 0x7fffffffLL) return cudaErrorInvalidValue;
    decode_split_kernel<<<dim3((unsigned)ctas, (unsigned)p.nsplit), DEC_THREADS, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<<<(unsigned)(L.B * L.Hq), kD, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace zgcm
