/*
 * zgcm_muon.h — C ABI of the Muon optimiser step for one matrix parameter (sm_100a).
 *
 * The optimiser the ZGCM-1 training system uses for its matrix parameters (ZGCM-1 summary,
 * section "前置知识 / Muon 优化器": momentum 0.9, spectral-norm scaling, five Newton–Schulz
 * iterations, learning rate 2e-4, weight decay 0.1, scalar parameters on Adam; shibing624
 * review, section "⚙️ 训练系统": momentum 0.9, 5 Newton–Schulz steps, constant learning rate
 * 2e-4).  For one m x n matrix W with gradient G and momentum buffer M:
 *
 *   M  <- momentum * M + G
 *   X0  = M / (||M||_F + eps)          (the Frobenius norm bounds the spectral norm: every
 *                                      singular value of X0 is at most 1)
 *   X  <- a X + (b A + c A A) X,  A = X X^T      (steps times, on the orientation with fewer
 *                                      rows: a tall M is transposed first and back after)
 *   W  <- W (1 - lr * weight_decay) - lr * X
 *
 * Readings where the pages are silent: plain momentum accumulation (no Nesterov term); the
 * Frobenius norm as the spectral-norm bound; the iteration's coefficients, which the pages do
 * not give — (a, b, c) = (1.5, -0.5, 0) is the classical Newton–Schulz step for the
 * orthogonal polar factor, and any other odd quintic may be passed; decoupled weight decay and
 * no further scale on the orthogonalised update.
 *
 * Precision: G, X and the iteration's products are bf16 operands with fp32 accumulation
 * (tcgen05.mma kind::f16); M and W are fp32; the norm is a fixed-order fp32 sum, so repeated
 * calls give the same bits.  Status codes: ZGCM_* of zgcm_attn.h.  All calls are asynchronous
 * on `cuda_stream` (NULL: the legacy default stream) and allocate nothing.
 *
 * Shapes: m, n >= 8 and multiples of 8 (row strides of 16 bytes for the TMA copies), m * n <
 * 2^40; steps in 0..100.  Tensors are row-major, 16-byte aligned, on the current device.
 */
#ifndef ZGCM_MUON_H
#define ZGCM_MUON_H

#include <stddef.h>

#include "zgcm_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of device workspace the two calls below need for an m x n matrix (0 for invalid
 * dimensions): two bf16 [p, q] iterates and two bf16 [p, p] products (p = min(m, n),
 * q = max(m, n)) and the norm's partial sums, each part 256-byte aligned. */
size_t zgcm_muon_workspace_size(int m, int n);

/*
 * One Muon step.  W fp32 [m, n] (updated in place), G bf16 [m, n] (read), M fp32 [m, n] (the
 * momentum buffer, updated in place).  workspace: at least zgcm_muon_workspace_size(m, n)
 * bytes, 256-byte aligned, contents on entry irrelevant, not shared with a concurrent call.
 * Returns ZGCM_ERR_INVALID_ARG (bad dimensions or steps, null pointer), ZGCM_ERR_ALIGNMENT,
 * ZGCM_ERR_WORKSPACE, ZGCM_ERR_CUDA; otherwise ZGCM_OK.
 */
int zgcm_muon_step(float* W, const void* G, float* M, int m, int n, float lr, float weight_decay, float momentum,
                   int steps, float a, float b, float c, float eps, void* workspace, size_t workspace_bytes,
                   void* cuda_stream);

/*
 * The orthogonalisation alone: out bf16 [m, n] = the iterate after `steps` iterations from
 * G / (||G||_F + eps), G bf16 [m, n].  Workspace and errors as zgcm_muon_step.
 */
int zgcm_muon_orthogonalize(const void* G, void* out, int m, int n, int steps, float a, float b, float c, float eps,
                            void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * The iteration's product kernel: C [M, N] = alpha * A op(B) + beta * D, bf16 A [M, K], C and
 * D [M, N] (D may be NULL: no beta term); B is [K, N] when b_kn = 1 (C = A B) and [N, K] when
 * b_kn = 0 (C = A B^T).  fp32 accumulation, one rounding to bf16.  N and K multiples of 8,
 * M >= 1.  C must not alias A, B or D.
 */
int zgcm_muon_gemm(const void* A, const void* B, const void* D, void* C, int M, int N, int K, float alpha,
                   float beta, int b_kn, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* ZGCM_MUON_H */
