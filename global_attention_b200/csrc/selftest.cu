// selftest.cu — the failure path of the bounded waits, exercised without a fault: one CTA
// waits on an mbarrier that nothing ever arrives on.  The wait gives up after its bound
// (kWaitLimit polls, about a second), the CTA records the site in the device error word
// exactly as the attention kernels do, and returns; the host then reads ZGCM_ERR_TIMEOUT
// through zgcm_attn_device_error and the context stays usable.
#include "sm100.cuh"

namespace zgcm {
using namespace sm100;

constexpr int kSelftestSite = 999;

__global__ void selftest_expired_wait_kernel(int* err) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        abort = 0;
        mbar_init(&bar, 1);   // one arrival expected; none will come
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile int* ab = &abort;
        if (!mbar_wait(&bar, 0, ab, kSelftestSite) && err) atomicExch(err, *ab);
    }
    __syncthreads();
}

cudaError_t launch_selftest_expired_wait(int* err_word, cudaStream_t stream) {
    selftest_expired_wait_kernel<<<1, 32, 0, stream>>>(err_word);
    return cudaGetLastError();
}

}  // namespace zgcm

// ------------------------------------------------------------------ MUFU exp2 rate probe

namespace zgcm {

// Each thread runs `iters` rounds of 8 independent exp2 chains (ex2.approx, the instruction
// the softmax kernels use) and stores their sum, so nothing is optimised away: 8 * iters
// exponentials per thread.  With enough warps the rate is the MUFU unit's throughput; with
// one warp per SM sub-partition it is one warp's latency-bound rate.
__global__ void probe_ex2_kernel(float* out, int iters) {
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = -1.0f - 0.001f * (threadIdx.x & 7) - 0.01f * k;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float y;
            asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(a[k]));
            a[k] = y - 1.5f;  // stays in (-1.5, -0.5): a bounded, data-dependent chain
        }
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += a[k];
    out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

cudaError_t launch_probe_ex2(float* out, int blocks, int threads, int iters, cudaStream_t stream) {
    probe_ex2_kernel<<<blocks, threads, 0, stream>>>(out, iters);
    return cudaGetLastError();
}

}  // namespace zgcm
