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
