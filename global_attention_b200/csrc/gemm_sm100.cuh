// gemm_sm100.cuh — the library's bf16 GEMM on tcgen05 / TMEM / TMA (sm_100a), for the Muon
// iterations and the projections around the attention layer:
//   C [M, N] = alpha * A B + beta * D      (logical A [M, K], B [K, N]; fp32 accumulation)
// with operands and result that may be split into up to four row-major tensors along one
// dimension (the q / k / v / g parts of a projection), so no caller has to concatenate.
#pragma once
#include <cuda_runtime.h>

#include "common.cuh"

namespace zgcm {

constexpr int GEMM_BM = 128;   // output rows of a CTA (MMA M)
constexpr int GEMM_BN = 256;   // output columns of a CTA (MMA N)
constexpr int GEMM_BK = 64;    // K of a pipeline stage
constexpr int GEMM_MAX_SEG = 4;

// One part of a split operand: a row-major bf16 tensor of rows x cols, whose first element
// along the split dimension is `start` of the whole.
struct GemmSeg {
    const void* ptr;
    int rows, cols;
    int start;
};

struct GemmDesc {
    int M, N, K;
    // A.  a_mn = 0: each part is [M, K_part] row-major (K contiguous); a_mn = 1: [K, M_part]
    // row-major (the transpose of A is stored).  a_split: 0 one part, 1 parts along K (a_mn = 0;
    // starts multiples of 64), 2 parts along M (a_mn = 1; starts multiples of 128).
    int a_mn = 0, a_split = 0, a_nseg = 1;
    GemmSeg a[GEMM_MAX_SEG];
    // B.  b_kn = 1: [K, N] row-major; 0: [N, K] row-major (C = A B^T)
    int b_kn = 0;
    const void* b = nullptr;
    // C: parts along N, c[s] row-major with leading dimension c_ld[s], its first column
    // c_start[s] (starts multiples of 256)
    int c_nseg = 1;
    void* c[GEMM_MAX_SEG] = {nullptr, nullptr, nullptr, nullptr};
    int c_ld[GEMM_MAX_SEG] = {0, 0, 0, 0};
    int c_start[GEMM_MAX_SEG] = {0, 0, 0, 0};
    const void* d = nullptr;  // [M, N] row-major beta term (one C part only), or null
    float alpha = 1.0f, beta = 0.0f;
    bool upper = false;       // C symmetric (M == N, one part): tiles wholly below the diagonal
                              // skipped, then that half copied from the other
};

// cudaErrorInvalidValue for a description the kernel does not take (the shape rules above,
// row strides of 16 bytes, 16-byte aligned tensors) or without the driver's tensor-map encoder.
cudaError_t launch_gemm(const GemmDesc& g, int* err_word, cudaStream_t stream);

}  // namespace zgcm
