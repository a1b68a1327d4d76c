// noalloc.cu — the backward without a caller-provided workspace.
//
// Some callers cannot allocate device memory: a process that reserved the whole GPU's
// memory for its own pool up front (a serving engine, say) has none left to hand out, a
// plugin interface may give its kernels no allocator at all, and cudaMalloc/cudaFree can
// synchronise the device, which latency-sensitive callers avoid.  For them the scratch
// lives in one file-scope device array of fixed size; this file is the only place that
// names it.
//
// The array exists on every GPU that loads this library and stays allocated until the
// process exits.  Every call on a device shares it and it keeps the last call's contents:
// the backward writes every scratch word it later reads (nothing in it must start at zero),
// and two calls whose executions overlap on the GPU — on different streams, or from
// different host threads — race on it.  The array used is the one of the calling thread's
// current device, so the tensors and the stream must belong to that device (a call whose q
// lives on another device is rejected with ZGCM_ERR_INVALID_ARG).
#include <mutex>

#include "zgcm_attn.h"

namespace {

constexpr size_t kScratchBytes = size_t(64) << 20;  // 64 MiB per device
static __device__ __align__(256) unsigned char zgcm_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch[kMaxDevices] = {};

// Device address of the scratch array on the current device (host code cannot use the
// array's name as a device address).  Looked up once per device, under a lock.
void* scratch_address(int* status) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *status = ZGCM_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, zgcm_noalloc_scratch) != cudaSuccess || !ptr) {
            *status = ZGCM_ERR_CUDA;
            return nullptr;
        }
        g_scratch[dev] = ptr;
    }
    *status = ZGCM_OK;
    return g_scratch[dev];
}

}  // namespace

extern "C" int zgcm_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* g,
                                     const float* gamma_q, const float* gamma_k,
                                     const void* out, const float* lse, const void* dout,
                                     int B, int S, int Hq, int Hkv, int D, int rope_dims,
                                     double rope_base, int window, int causal, float eps, float scale,
                                     void* dq, void* dk, void* dv, void* dg,
                                     float* dgamma_q, float* dgamma_k, void* cuda_stream) {
    const size_t need = zgcm_attn_bwd_workspace_size(B, S, Hq, Hkv, D, window);
    if (need > kScratchBytes) return ZGCM_ERR_TOO_LARGE;
    void* ws = nullptr;
    if ((long long)B * S > 0) {
        const void* ptrs[] = {q, k, v, g, gamma_q, gamma_k, out, lse, dout, dq, dk, dv, dg, dgamma_q, dgamma_k};
        for (const void* p : ptrs)
            if (!p) return ZGCM_ERR_INVALID_ARG;
        // The scratch used is the current device's: the tensors must live there too.
        int dev = 0;
        cudaPointerAttributes attr;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaPointerGetAttributes(&attr, q) != cudaSuccess)
            return ZGCM_ERR_CUDA;
        if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return ZGCM_ERR_INVALID_ARG;
        if (attr.device != dev) return ZGCM_ERR_INVALID_ARG;
        int st = ZGCM_OK;
        ws = scratch_address(&st);
        if (st != ZGCM_OK) return st;
    }
    return zgcm_attn_bwd(q, k, v, g, gamma_q, gamma_k, out, lse, dout, B, S, Hq, Hkv, D, rope_dims, rope_base,
                         window, causal, eps, scale, dq, dk, dv, dg, dgamma_q, dgamma_k, ws, kScratchBytes,
                         cuda_stream);
}
