/*
 * zgcm_proj.h — C ABI of the projections around the gated attention layer (sm_100a), bf16.
 *
 * The layer's inputs q, k, v and the gate logits g are linear projections of the layer input,
 * and its output goes through an output projection (ZGCM-1: hidden size 4096, 32 query / 8
 * KV heads of 128, ZGCM-1 summary, section "核心方法"; matrix products in mixed FP8 through
 * the training system's GEMMs, shibing624 review, section "⚙️ 训练系统").  Readings: the gate
 * logits come from their own linear map of the layer input (the pages do not say where g
 * comes from); no biases; bf16 operands and results with fp32 accumulation (the FP8 E4M3 /
 * E5M2 variant with delayed scaling that the pages describe is not built).
 *
 * Layouts (row-major, T = B*S tokens, the attention calls' [B,S,H,D] tensors are [T, H*D]):
 *   x [T, d_model];  W_qkvg [(2*Hq + 2*Hkv)*D, d_model], the rows of W_q, W_k, W_v, W_g in
 *   that order (the layout of a torch Linear's weight, out_features x in_features);
 *   q, g [T, Hq*D];  k, v [T, Hkv*D];  attention output a [T, d_in];  W_o [d_model, d_in];
 *   y [T, d_model].
 * Forward:   q|k|v|g = x W_qkvg^T        y = a W_o^T
 * Backward:  dx = [dq|dk|dv|dg] W_qkvg   dW_qkvg = [dq|dk|dv|dg]^T x
 *            da = dy W_o                 dW_o = dy^T a
 * (weight gradients overwritten, not accumulated, in bf16).  One tcgen05 GEMM per product
 * (gemm_sm100.cu): the split outputs and operands are read and written in place, never
 * concatenated.
 *
 * Requirements: T >= 1 (any value); d_model, d_in, Hq*D, Hkv*D multiples of 256 (so that every output
 * part starts on a 256-column tile and every split operand on a 128-row one); 16-byte
 * aligned tensors; outputs not aliasing inputs.  Errors: ZGCM_ERR_INVALID_ARG (null pointer,
 * bad shape), ZGCM_ERR_ALIGNMENT, ZGCM_ERR_CUDA.  Asynchronous on `cuda_stream`; nothing is
 * allocated.
 */
#ifndef ZGCM_PROJ_H
#define ZGCM_PROJ_H

#include "zgcm_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

int zgcm_proj_qkvg_fwd(const void* x, const void* w_qkvg, int T, int d_model, int Hq, int Hkv, int D, void* q,
                       void* k, void* v, void* g, void* cuda_stream);
int zgcm_proj_qkvg_bwd(const void* x, const void* w_qkvg, const void* dq, const void* dk, const void* dv,
                       const void* dg, int T, int d_model, int Hq, int Hkv, int D, void* dx, void* dw_qkvg,
                       void* cuda_stream);
int zgcm_proj_out_fwd(const void* a, const void* w_o, int T, int d_in, int d_model, void* y, void* cuda_stream);
int zgcm_proj_out_bwd(const void* a, const void* w_o, const void* dy, int T, int d_in, int d_model, void* da,
                      void* dw_o, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* ZGCM_PROJ_H */
