// zgcm_attn.cu — the C ABI (include/zgcm_attn.h): argument checks, parameter set-up,
// workspace layout and kernel launches.  Host code only; the kernels live in the other
// .cu files of this directory.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include "zgcm_attn.h"
#include "common.cuh"

namespace zgcm {
cudaError_t launch_fwd_tc(const FwdParams& p, void* workspace, int* err_word, cudaStream_t stream,
                          const SavedAct* sv);
bool fwd_tc_supported(const LayerParams& L);
cudaError_t launch_fwd_strip(const FwdParams& fp, int* err_word, cudaStream_t stream, const SavedAct* sv);
bool fwd_strip_supported(const LayerParams& L);
cudaError_t launch_fwd_glob_tc(const FwdParams& p, void* workspace, int* err_word, cudaStream_t stream,
                               const SavedAct* sv);
bool fwd_glob_supported(const LayerParams& L);
size_t decode_workspace_bytes(int B, int Hq, int window, int C);
cudaError_t launch_selftest_expired_wait(int* err_word, cudaStream_t stream);
cudaError_t launch_decode(const LayerParams& L, const int* pos, void* k_cache, void* v_cache, int C, void* out,
                          float* lse, void* workspace, cudaStream_t stream);
size_t fwd_glob_workspace_bytes(int B, int S, int Hkv);
cudaError_t launch_bwd_tc(const BwdParams& bp, void* workspace, int* err_word, cudaStream_t stream,
                          void* const* events, int n_pairs, const SavedAct* sv);
extern const char* const kBwdTcSavedKernelNames[];
extern const int kBwdTcSavedKernelCount;
extern const char* const kBwdWideSavedKernelNames[];
extern const int kBwdWideSavedKernelCount;
bool bwd_tc_supported(const LayerParams& L);
bool bwd_wide_supported(const LayerParams& L);
extern const char* const kBwdWideKernelNames[];
extern const int kBwdWideKernelCount;
size_t bwd_tc_workspace_bytes(int B, int S, int Hq, int Hkv);
extern const char* const kBwdTcKernelNames[];
extern const int kBwdTcKernelCount;
}  // namespace zgcm

using namespace zgcm;

// Site of the last bounded device wait that expired (0 = none); read and cleared by
// zgcm_attn_device_error().  Written only on a failure path.
__device__ int zgcm_device_error_word;

namespace {

int* device_error_word() {
    void* ptr = nullptr;
    return cudaGetSymbolAddress(&ptr, zgcm_device_error_word) == cudaSuccess ? static_cast<int*>(ptr) : nullptr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace zgcm {
// the error word for the library's other kernels (the Muon step)
int* library_error_word() { return device_error_word(); }
}  // namespace zgcm

namespace {

// Forward kernel for a layer: the strip kernel (W <= 128, 4 query heads per KV head), the
// sliding-window tcgen05 kernel (W <= 128, other group sizes) or the wide-window / global
// tcgen05 pair (W > 128).  Every shape the arguments allow has one of them.
enum class FwdPath { STRIP, TC, GLOB };

FwdPath fwd_path(const LayerParams& L) {
    if (fwd_strip_supported(L)) return FwdPath::STRIP;
    if (fwd_tc_supported(L)) return FwdPath::TC;
    return FwdPath::GLOB;
}

LayerParams shape_only(int B, int S, int Hq, int Hkv, int rope_dims, int window) {
    LayerParams L{};
    L.B = B; L.S = S; L.Hq = Hq; L.Hkv = Hkv; L.G = Hkv > 0 ? Hq / Hkv : 0;
    L.rope_half = rope_dims / 2; L.W = window;
    return L;
}

// Checks shared by forward and backward.  Returns ZGCM_OK or the first failing status.
int check_shape(int B, int S, int Hq, int Hkv, int D, int rope_dims, double rope_base, int window,
                int causal, float eps, float scale) {
    if (B < 0 || S < 0 || Hq < 1 || Hkv < 1 || D < 1) return ZGCM_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ZGCM_ERR_INVALID_ARG;
    if (rope_dims < 0 || rope_dims > D || (rope_dims & 1)) return ZGCM_ERR_INVALID_ARG;
    if (rope_dims > 0 && !(rope_base > 0.0 && isfinite(rope_base))) return ZGCM_ERR_INVALID_ARG;
    if (window < 1) return ZGCM_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return ZGCM_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return ZGCM_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ZGCM_ERR_INVALID_ARG;
    if (causal == 0) return ZGCM_ERR_UNSUPPORTED;  // the pages describe causal layers only
    if (D != kD) return ZGCM_ERR_UNSUPPORTED;
    if ((long double)B * S * Hq * D >= (long double)(1ULL << 40)) return ZGCM_ERR_UNSUPPORTED;
    return ZGCM_OK;
}

void fill_layer(LayerParams& L, const void* q, const void* k, const void* v, const void* g,
                const float* gamma_q, const float* gamma_k, int B, int S, int Hq, int Hkv,
                int rope_dims, double rope_base, int window, float eps, float scale) {
    L.q = static_cast<const bf16*>(q);
    L.k = static_cast<const bf16*>(k);
    L.v = static_cast<const bf16*>(v);
    L.g = static_cast<const bf16*>(g);
    L.gamma_q = gamma_q;
    L.gamma_k = gamma_k;
    L.B = B; L.S = S; L.Hq = Hq; L.Hkv = Hkv; L.G = Hq / Hkv;
    L.rope_half = rope_dims / 2;
    L.W = window;
    L.q_off = 0;
    L.Sq = S;
    L.eps = eps;
    L.scale = scale;
    L.scale_log2 = scale * kLog2e;
    for (int t = 0; t < kMaxHalf; ++t)
        L.theta[t] = t < L.rope_half ? pow(rope_base, -2.0 * (double)t / (double)rope_dims) : 0.0;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The activation store a forward leaves for the backward: Q~ fp16 [B,S,Hq,D], the q rows'
// inverse RMS fp32 [B,Hq,S], K~ fp16 [B,S,Hkv,D] (the forward's own K~ workspace) and the k
// rows' inverse RMS fp32 [B,Hkv,S], each 256-byte aligned.
size_t saved_layout(int B, int S, int Hq, int Hkv, char* base, SavedAct* sv) {
    const size_t rows = (size_t)B * S * Hq, krows = (size_t)B * S * Hkv;
    size_t off = 0;
    const size_t q16 = off;   off = align256(off + rows * kD * 2);
    const size_t qrinv = off; off = align256(off + rows * 4);
    const size_t k16 = off;   off = align256(off + krows * kD * 2);
    const size_t krinv = off; off = align256(off + krows * 4);
    if (sv) {
        sv->q16 = base + q16;
        sv->qrinv = reinterpret_cast<float*>(base + qrinv);
        sv->k16 = base + k16;
        sv->krinv = reinterpret_cast<float*>(base + krinv);
    }
    return off;
}

// The store applies to every shape (both passes run tcgen05 kernels throughout).
bool saved_supported(const LayerParams& L) { return L.S >= 1 && L.B >= 1; }

// Query rows Sq at the end of S key rows (the first at position q_off = S - Sq): every Sq
// with q_off = 0, else q_off a multiple of 128 and a window wider than 128 (the wide-window
// kernels take the offset; a window of at most 128 reaches 127 rows back, so a caller pads
// those few rows instead).
int rows_check(int S, int Sq, int window) {
    if (Sq < 0 || Sq > S) return ZGCM_ERR_INVALID_ARG;
    const int q_off = S - Sq;
    if (q_off == 0) return ZGCM_OK;
    if (q_off % 128 != 0 || window <= 128) return ZGCM_ERR_UNSUPPORTED;
    return ZGCM_OK;
}

}  // namespace

extern "C" {

const char* zgcm_status_string(int status) {
    switch (status) {
        case ZGCM_OK: return "ZGCM_OK";
        case ZGCM_ERR_INVALID_ARG: return "ZGCM_ERR_INVALID_ARG: invalid argument";
        case ZGCM_ERR_UNSUPPORTED: return "ZGCM_ERR_UNSUPPORTED: valid but unsupported configuration";
        case ZGCM_ERR_ALIGNMENT: return "ZGCM_ERR_ALIGNMENT: tensor pointer not 16-byte aligned";
        case ZGCM_ERR_WORKSPACE: return "ZGCM_ERR_WORKSPACE: workspace missing or too small";
        case ZGCM_ERR_CUDA: return "ZGCM_ERR_CUDA: CUDA runtime or launch failure";
        case ZGCM_ERR_TIMEOUT: return "ZGCM_ERR_TIMEOUT: bounded device wait expired";
        case ZGCM_ERR_TOO_LARGE:
            return "ZGCM_ERR_TOO_LARGE: problem needs more than the 64 MiB scratch of zgcm_attn_bwd_noalloc";
        default: return "unknown zgcm_status";
    }
}

size_t zgcm_attn_fwd_workspace_size(int B, int S, int Hq, int Hkv, int D, int rope_dims, int window) {
    if (check_shape(B, S, Hq, Hkv, D, rope_dims, 1.0, window, 1, 0.f, 1.f) != ZGCM_OK) return 0;
    if ((long long)B * S == 0) return 0;
    // the tcgen05 forwards other than the strip kernel read K~ (fp16, normalised and rotated
    // once per key tile) from it; the strip kernel normalises its key chunks in shared memory
    const FwdPath f = fwd_path(shape_only(B, S, Hq, Hkv, rope_dims, window));
    return f != FwdPath::STRIP ? align256(fwd_glob_workspace_bytes(B, S, Hkv)) : 0;
}

}  // extern "C"

namespace {
// Checks of the forward's arguments other than the workspace (ZGCM_OK or the first failure).
int fwd_check(const void* q, const void* k, const void* v, const void* g, const float* gamma_q,
              const float* gamma_k, int B, int S, int Hq, int Hkv, int D, int rope_dims, double rope_base,
              int window, int causal, float eps, float scale, const void* out, const float* lse) {
    int st = check_shape(B, S, Hq, Hkv, D, rope_dims, rope_base, window, causal, eps, scale);
    if (st != ZGCM_OK || (long long)B * S == 0) return st;
    const void* ptrs[] = {q, k, v, g, gamma_q, gamma_k, out, lse};
    for (const void* p : ptrs)
        if (!p) return ZGCM_ERR_INVALID_ARG;
    for (const void* p : ptrs)
        if (!aligned16(p)) return ZGCM_ERR_ALIGNMENT;
    return ZGCM_OK;
}
}  // namespace

extern "C" {

int zgcm_attn_fwd_ws(const void* q, const void* k, const void* v, const void* g,
                     const float* gamma_q, const float* gamma_k,
                     int B, int S, int Hq, int Hkv, int D, int rope_dims,
                     double rope_base, int window, int causal, float eps, float scale,
                     void* out, float* lse, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    int st = fwd_check(q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, D, rope_dims, rope_base, window, causal,
                       eps, scale, out, lse);
    if (st != ZGCM_OK) return st;
    if ((long long)B * S == 0) return ZGCM_OK;
    const size_t need = zgcm_attn_fwd_workspace_size(B, S, Hq, Hkv, D, rope_dims, window);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return ZGCM_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ZGCM_ERR_ALIGNMENT;
    }
    FwdParams p;
    fill_layer(p.L, q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, rope_dims, rope_base, window, eps, scale);
    p.out = static_cast<bf16*>(out);
    p.lse = lse;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    cudaError_t e;
    switch (fwd_path(p.L)) {
        case FwdPath::STRIP: e = launch_fwd_strip(p, device_error_word(), stream, nullptr); break;
        case FwdPath::TC: e = launch_fwd_tc(p, workspace, device_error_word(), stream, nullptr); break;
        default: e = launch_fwd_glob_tc(p, workspace, device_error_word(), stream, nullptr); break;
    }
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}

int zgcm_attn_fwd(const void* q, const void* k, const void* v, const void* g,
                  const float* gamma_q, const float* gamma_k,
                  int B, int S, int Hq, int Hkv, int D, int rope_dims,
                  double rope_base, int window, int causal, float eps, float scale,
                  void* out, float* lse, void* cuda_stream) {
    const int st0 = fwd_check(q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, D, rope_dims, rope_base, window,
                              causal, eps, scale, out, lse);
    if (st0 != ZGCM_OK) return st0;
    const size_t need = zgcm_attn_fwd_workspace_size(B, S, Hq, Hkv, D, rope_dims, window);
    if (need == 0)
        return zgcm_attn_fwd_ws(q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, D, rope_dims, rope_base, window,
                                causal, eps, scale, out, lse, nullptr, 0, cuda_stream);
    // stream-ordered scratch: taken from and returned to the device's default memory pool
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    void* ws = nullptr;
    if (cudaMallocAsync(&ws, need, stream) != cudaSuccess) return ZGCM_ERR_CUDA;
    const int st = zgcm_attn_fwd_ws(q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, D, rope_dims, rope_base,
                                    window, causal, eps, scale, out, lse, ws, need, cuda_stream);
    const cudaError_t e = cudaFreeAsync(ws, stream);
    if (st != ZGCM_OK) return st;
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}

int zgcm_attn_fwd_rows(const void* q, const void* k, const void* v, const void* g,
                       const float* gamma_q, const float* gamma_k,
                       int B, int Sq, int S, int Hq, int Hkv, int D, int rope_dims,
                       double rope_base, int window, int causal, float eps, float scale,
                       void* out, float* lse, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    int st = check_shape(B, S, Hq, Hkv, D, rope_dims, rope_base, window, causal, eps, scale);
    if (st != ZGCM_OK) return st;
    if ((st = rows_check(S, Sq, window)) != ZGCM_OK) return st;
    if ((long long)B * Sq == 0) return ZGCM_OK;  // no query row: nothing to compute
    if (Sq == S)
        return zgcm_attn_fwd_ws(q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, D, rope_dims, rope_base, window,
                                causal, eps, scale, out, lse, workspace, workspace_bytes, cuda_stream);
    st = fwd_check(q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, D, rope_dims, rope_base, window, causal, eps, scale,
                   out, lse);
    if (st != ZGCM_OK) return st;
    const size_t need = zgcm_attn_fwd_workspace_size(B, S, Hq, Hkv, D, rope_dims, window);
    if (!workspace || workspace_bytes < need) return ZGCM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ZGCM_ERR_ALIGNMENT;
    FwdParams p;
    fill_layer(p.L, q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, rope_dims, rope_base, window, eps, scale);
    p.L.q_off = S - Sq;
    p.L.Sq = Sq;
    p.out = static_cast<bf16*>(out);
    p.lse = lse;
    const cudaError_t e =
        launch_fwd_glob_tc(p, workspace, device_error_word(), static_cast<cudaStream_t>(cuda_stream), nullptr);
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}

size_t zgcm_attn_saved_size(int B, int S, int Hq, int Hkv, int D, int rope_dims, int window) {
    if (check_shape(B, S, Hq, Hkv, D, rope_dims, 1.0, window, 1, 0.f, 1.f) != ZGCM_OK) return 0;
    if ((long long)B * S == 0) return 0;
    if (!saved_supported(shape_only(B, S, Hq, Hkv, rope_dims, window))) return 0;
    return saved_layout(B, S, Hq, Hkv, nullptr, nullptr);
}

int zgcm_attn_fwd_save(const void* q, const void* k, const void* v, const void* g,
                       const float* gamma_q, const float* gamma_k,
                       int B, int S, int Hq, int Hkv, int D, int rope_dims,
                       double rope_base, int window, int causal, float eps, float scale,
                       void* out, float* lse, void* saved, size_t saved_bytes, void* cuda_stream) {
    int st = fwd_check(q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, D, rope_dims, rope_base, window, causal,
                       eps, scale, out, lse);
    if (st != ZGCM_OK) return st;
    if ((long long)B * S == 0) return ZGCM_OK;
    FwdParams p;
    fill_layer(p.L, q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, rope_dims, rope_base, window, eps, scale);
    if (!saved_supported(p.L)) return ZGCM_ERR_UNSUPPORTED;
    if (!saved || saved_bytes < zgcm_attn_saved_size(B, S, Hq, Hkv, D, rope_dims, window)) return ZGCM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(saved) & 255u) return ZGCM_ERR_ALIGNMENT;
    SavedAct sv;
    saved_layout(B, S, Hq, Hkv, static_cast<char*>(saved), &sv);
    p.out = static_cast<bf16*>(out);
    p.lse = lse;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    const FwdPath f = fwd_path(p.L);
    const cudaError_t e = f == FwdPath::STRIP ? launch_fwd_strip(p, device_error_word(), stream, &sv)
                          : f == FwdPath::TC  ? launch_fwd_tc(p, sv.k16, device_error_word(), stream, &sv)
                                              : launch_fwd_glob_tc(p, sv.k16, device_error_word(), stream, &sv);
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}

size_t zgcm_attn_decode_workspace_size(int B, int Hq, int window, int cache_len) {
    if (B <= 0 || Hq < 1 || window < 1 || cache_len < 1) return 0;
    return decode_workspace_bytes(B, Hq, window, cache_len);
}

int zgcm_attn_decode(const void* q, const void* k, const void* v, const void* g,
                     const float* gamma_q, const float* gamma_k, const int* pos,
                     int B, int Hq, int Hkv, int D, int rope_dims, double rope_base, int window,
                     float eps, float scale, void* k_cache, void* v_cache, int cache_len,
                     void* out, float* lse, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    int st = check_shape(B, 1, Hq, Hkv, D, rope_dims, rope_base, window, 1, eps, scale);
    if (st != ZGCM_OK) return st;
    if (cache_len < 1) return ZGCM_ERR_INVALID_ARG;
    if (B == 0) return ZGCM_OK;
    if ((long double)B * cache_len * Hkv * D >= (long double)(1ULL << 40)) return ZGCM_ERR_UNSUPPORTED;
    const void* ptrs[] = {q, k, v, g, gamma_q, gamma_k, pos, k_cache, v_cache, out, lse};
    for (const void* p : ptrs)
        if (!p) return ZGCM_ERR_INVALID_ARG;
    for (const void* p : ptrs)
        if (!aligned16(p)) return ZGCM_ERR_ALIGNMENT;
    const size_t need = zgcm_attn_decode_workspace_size(B, Hq, window, cache_len);
    if (!workspace || workspace_bytes < need) return ZGCM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ZGCM_ERR_ALIGNMENT;
    LayerParams L;
    fill_layer(L, q, k, v, g, gamma_q, gamma_k, B, 1, Hq, Hkv, rope_dims, rope_base, window, eps, scale);
    const cudaError_t e = launch_decode(L, static_cast<const int*>(pos), k_cache, v_cache, cache_len, out, lse,
                                        workspace, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}

int zgcm_attn_selftest_expired_wait(void* cuda_stream) {
    return launch_selftest_expired_wait(device_error_word(), static_cast<cudaStream_t>(cuda_stream)) == cudaSuccess
               ? ZGCM_OK
               : ZGCM_ERR_CUDA;
}

int zgcm_attn_device_error(void) {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, zgcm_device_error_word, sizeof(int)) != cudaSuccess) return ZGCM_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(zgcm_device_error_word, &zero, sizeof(int)) != cudaSuccess) return ZGCM_ERR_CUDA;
    return v == 0 ? ZGCM_OK : ZGCM_ERR_TIMEOUT;
}

const char* zgcm_attn_fwd_kernel_name(int B, int S, int Hq, int Hkv, int rope_dims, int window) {
    switch (fwd_path(shape_only(B, S, Hq, Hkv, rope_dims, window))) {
        case FwdPath::STRIP: return "fwd_strip_kernel";
        case FwdPath::TC: return "fwd_tc_kernel";
        default: return "fwd_glob_tc_kernel";
    }
}

size_t zgcm_attn_bwd_workspace_size(int B, int S, int Hq, int Hkv, int D, int window) {
    if (check_shape(B, S, Hq, Hkv, D, 0, 1.0, window, 1, 0.f, 1.f) != ZGCM_OK) return 0;
    if ((long long)B * S == 0) return 0;
    return bwd_tc_workspace_bytes(B, S, Hq, Hkv);
}

}  // extern "C"

namespace {
// The backward; with `saved` (non-null), from the activations zgcm_attn_fwd_save left there.
// Sq: the query rows (the last Sq of the S positions; Sq = S for every other entry).
int bwd_run(const void* q, const void* k, const void* v, const void* g, const float* gamma_q,
            const float* gamma_k, const void* out, const float* lse, const void* dout, int B, int Sq, int S, int Hq,
            int Hkv, int D, int rope_dims, double rope_base, int window, int causal, float eps, float scale,
            void* dq, void* dk, void* dv, void* dg, float* dgamma_q, float* dgamma_k, void* workspace,
            size_t workspace_bytes, const void* saved, size_t saved_bytes, void* cuda_stream,
            void* const* events, int n_pairs) {
    int st = check_shape(B, S, Hq, Hkv, D, rope_dims, rope_base, window, causal, eps, scale);
    if (st != ZGCM_OK) return st;
    if ((st = rows_check(S, Sq, window)) != ZGCM_OK) return st;
    if (saved && Sq != S) return ZGCM_ERR_UNSUPPORTED;
    if (!dgamma_q || !dgamma_k) return ZGCM_ERR_INVALID_ARG;
    if (!aligned16(dgamma_q) || !aligned16(dgamma_k)) return ZGCM_ERR_ALIGNMENT;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if ((long long)B * Sq == 0) {
        // no query row: zero key gradients (when there are key rows) and d_gamma
        if ((long long)B * S > 0) {
            if (!dk || !dv) return ZGCM_ERR_INVALID_ARG;
            if (!aligned16(dk) || !aligned16(dv)) return ZGCM_ERR_ALIGNMENT;
            const size_t kv_bytes = (size_t)B * S * Hkv * kD * sizeof(bf16);
            if (cudaMemsetAsync(dk, 0, kv_bytes, stream) != cudaSuccess) return ZGCM_ERR_CUDA;
            if (cudaMemsetAsync(dv, 0, kv_bytes, stream) != cudaSuccess) return ZGCM_ERR_CUDA;
        }
        if (cudaMemsetAsync(dgamma_q, 0, kD * sizeof(float), stream) != cudaSuccess) return ZGCM_ERR_CUDA;
        if (cudaMemsetAsync(dgamma_k, 0, kD * sizeof(float), stream) != cudaSuccess) return ZGCM_ERR_CUDA;
        return ZGCM_OK;
    }
    const void* ptrs[] = {q, k, v, g, gamma_q, gamma_k, out, lse, dout, dq, dk, dv, dg};
    for (const void* p : ptrs)
        if (!p) return ZGCM_ERR_INVALID_ARG;
    for (const void* p : ptrs)
        if (!aligned16(p)) return ZGCM_ERR_ALIGNMENT;
    const size_t need = zgcm_attn_bwd_workspace_size(B, S, Hq, Hkv, D, window);
    if (!workspace || workspace_bytes < need) return ZGCM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ZGCM_ERR_ALIGNMENT;

    BwdParams p;
    fill_layer(p.L, q, k, v, g, gamma_q, gamma_k, B, S, Hq, Hkv, rope_dims, rope_base, window, eps, scale);
    p.L.q_off = S - Sq;
    p.L.Sq = Sq;
    p.out = static_cast<const bf16*>(out);
    p.lse = lse;
    p.dout = static_cast<const bf16*>(dout);
    p.dq = static_cast<bf16*>(dq);
    p.dk = static_cast<bf16*>(dk);
    p.dv = static_cast<bf16*>(dv);
    p.dg = static_cast<bf16*>(dg);
    p.dgamma_q = dgamma_q;
    p.dgamma_k = dgamma_k;
    if (n_pairs < 0 || (n_pairs > 0 && !events)) return ZGCM_ERR_INVALID_ARG;
    SavedAct sv;
    if (saved) {
        if (!saved_supported(p.L)) return ZGCM_ERR_UNSUPPORTED;
        if (saved_bytes < saved_layout(B, S, Hq, Hkv, nullptr, nullptr)) return ZGCM_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(saved) & 255u) return ZGCM_ERR_ALIGNMENT;
        saved_layout(B, S, Hq, Hkv, static_cast<char*>(const_cast<void*>(saved)), &sv);
    }
    const cudaError_t e =
        launch_bwd_tc(p, workspace, device_error_word(), stream, events, n_pairs, saved ? &sv : nullptr);
    return e == cudaSuccess ? ZGCM_OK : ZGCM_ERR_CUDA;
}
}  // namespace

extern "C" {

int zgcm_attn_bwd_timed(const void* q, const void* k, const void* v, const void* g,
                        const float* gamma_q, const float* gamma_k,
                        const void* out, const float* lse, const void* dout,
                        int B, int S, int Hq, int Hkv, int D, int rope_dims,
                        double rope_base, int window, int causal, float eps, float scale,
                        void* dq, void* dk, void* dv, void* dg,
                        float* dgamma_q, float* dgamma_k,
                        void* workspace, size_t workspace_bytes, void* cuda_stream,
                        void* const* events, int n_pairs) {
    return bwd_run(q, k, v, g, gamma_q, gamma_k, out, lse, dout, B, S, S, Hq, Hkv, D, rope_dims, rope_base,
                   window, causal, eps, scale, dq, dk, dv, dg, dgamma_q, dgamma_k, workspace, workspace_bytes, nullptr,
                   0, cuda_stream, events, n_pairs);
}

int zgcm_attn_bwd_rows(const void* q, const void* k, const void* v, const void* g,
                       const float* gamma_q, const float* gamma_k,
                       const void* out, const float* lse, const void* dout,
                       int B, int Sq, int S, int Hq, int Hkv, int D, int rope_dims,
                       double rope_base, int window, int causal, float eps, float scale,
                       void* dq, void* dk, void* dv, void* dg,
                       float* dgamma_q, float* dgamma_k,
                       void* workspace, size_t workspace_bytes, void* cuda_stream) {
    return bwd_run(q, k, v, g, gamma_q, gamma_k, out, lse, dout, B, Sq, S, Hq, Hkv, D, rope_dims, rope_base,
                   window, causal, eps, scale, dq, dk, dv, dg, dgamma_q, dgamma_k, workspace, workspace_bytes, nullptr,
                   0, cuda_stream, nullptr, 0);
}

int zgcm_attn_bwd_saved(const void* q, const void* k, const void* v, const void* g,
                        const float* gamma_q, const float* gamma_k,
                        const void* out, const float* lse, const void* dout,
                        int B, int S, int Hq, int Hkv, int D, int rope_dims,
                        double rope_base, int window, int causal, float eps, float scale,
                        void* dq, void* dk, void* dv, void* dg,
                        float* dgamma_q, float* dgamma_k,
                        void* workspace, size_t workspace_bytes, const void* saved, size_t saved_bytes,
                        void* cuda_stream, void* const* events, int n_pairs) {
    if (!saved) return ZGCM_ERR_INVALID_ARG;
    return bwd_run(q, k, v, g, gamma_q, gamma_k, out, lse, dout, B, S, S, Hq, Hkv, D, rope_dims, rope_base,
                   window, causal, eps, scale, dq, dk, dv, dg, dgamma_q, dgamma_k, workspace, workspace_bytes, saved,
                   saved_bytes, cuda_stream, events, n_pairs);
}

const char* zgcm_attn_bwd_saved_kernel_name(int i, int S, int rope_dims, int window) {
    LayerParams L{};
    L.B = 1; L.S = S; L.rope_half = rope_dims / 2; L.W = window;
    const char* const* names = nullptr;
    int n = 0;
    if (S >= 1 && bwd_tc_supported(L)) {
        names = kBwdTcSavedKernelNames;
        n = kBwdTcSavedKernelCount;
    } else if (S >= 1 && bwd_wide_supported(L)) {
        names = kBwdWideSavedKernelNames;
        n = kBwdWideSavedKernelCount;
    }
    return (i >= 0 && i < n) ? names[i] : nullptr;
}

const char* zgcm_attn_bwd_kernel_name(int i, int S, int rope_dims, int window) {
    LayerParams L{};
    L.B = 1; L.S = S; L.rope_half = rope_dims / 2; L.W = window;
    const char* const* names = nullptr;
    int n = 0;
    if (S >= 1 && bwd_tc_supported(L)) {
        names = kBwdTcKernelNames;
        n = kBwdTcKernelCount;
    } else if (S >= 1 && bwd_wide_supported(L)) {
        names = kBwdWideKernelNames;
        n = kBwdWideKernelCount;
    }
    return (i >= 0 && i < n) ? names[i] : nullptr;
}

int zgcm_attn_bwd(const void* q, const void* k, const void* v, const void* g,
                  const float* gamma_q, const float* gamma_k,
                  const void* out, const float* lse, const void* dout,
                  int B, int S, int Hq, int Hkv, int D, int rope_dims,
                  double rope_base, int window, int causal, float eps, float scale,
                  void* dq, void* dk, void* dv, void* dg,
                  float* dgamma_q, float* dgamma_k,
                  void* workspace, size_t workspace_bytes, void* cuda_stream) {
    return zgcm_attn_bwd_timed(q, k, v, g, gamma_q, gamma_k, out, lse, dout, B, S, Hq, Hkv, D,
                               rope_dims, rope_base, window, causal, eps, scale, dq, dk, dv, dg,
                               dgamma_q, dgamma_k, workspace, workspace_bytes, cuda_stream,
                               nullptr, 0);
}

}  // extern "C"
