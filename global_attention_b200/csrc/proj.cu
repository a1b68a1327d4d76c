// proj.cu — the C ABI of include/zgcm_proj.h: argument checks and the GEMM descriptions of the
// projections around the attention layer, each one launch of the library's tcgen05 GEMM
// (gemm_sm100.cu) with the q / k / v / g parts split in place.
#include <stdint.h>

#include "zgcm_proj.h"
#include "gemm_sm100.cuh"

namespace zgcm {
int* library_error_word();  // zgcm_attn.cu: the site of an expired bounded wait
}

using namespace zgcm;

namespace {

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_widths(int T, std::initializer_list<int> widths) {
    if (T < 1) return ZGCM_ERR_INVALID_ARG;
    for (int w : widths)
        if (w < 256 || w % 256 != 0) return ZGCM_ERR_INVALID_ARG;
    return ZGCM_OK;
}

int check_ptrs(std::initializer_list<const void*> ptrs) {
    for (const void* p : ptrs)
        if (!p) return ZGCM_ERR_INVALID_ARG;
    for (const void* p : ptrs)
        if (!aligned16(p)) return ZGCM_ERR_ALIGNMENT;
    return ZGCM_OK;
}

int run(const GemmDesc& g, void* stream) {
    return launch_gemm(g, library_error_word(), static_cast<cudaStream_t>(stream)) == cudaSuccess ? ZGCM_OK
                                                                                                  : ZGCM_ERR_CUDA;
}

}  // namespace

extern "C" {

int zgcm_proj_qkvg_fwd(const void* x, const void* w_qkvg, int T, int d_model, int Hq, int Hkv, int D, void* q,
                       void* k, void* v, void* g, void* cuda_stream) {
    const long long wq = (long long)Hq * D, wkv = (long long)Hkv * D;
    if (Hq < 1 || Hkv < 1 || D < 1 || 2 * (wq + wkv) > (1 << 30)) return ZGCM_ERR_INVALID_ARG;
    int st = check_widths(T, {d_model, (int)wq, (int)wkv});
    if (st == ZGCM_OK) st = check_ptrs({x, w_qkvg, q, k, v, g});
    if (st != ZGCM_OK) return st;
    // C [T, 2wq + 2wkv] = x W^T, its columns in four parts
    GemmDesc d;
    d.M = T;
    d.N = (int)(2 * (wq + wkv));
    d.K = d_model;
    d.a[0] = GemmSeg{x, T, d_model, 0};
    d.b_kn = 0;
    d.b = w_qkvg;
    d.c_nseg = 4;
    void* parts[4] = {q, k, v, g};
    const int width[4] = {(int)wq, (int)wkv, (int)wkv, (int)wq};
    int start = 0;
    for (int s = 0; s < 4; ++s) {
        d.c[s] = parts[s];
        d.c_ld[s] = width[s];
        d.c_start[s] = start;
        start += width[s];
    }
    return run(d, cuda_stream);
}

int zgcm_proj_qkvg_bwd(const void* x, const void* w_qkvg, const void* dq, const void* dk, const void* dv,
                       const void* dg, int T, int d_model, int Hq, int Hkv, int D, void* dx, void* dw_qkvg,
                       void* cuda_stream) {
    const long long wq = (long long)Hq * D, wkv = (long long)Hkv * D;
    if (Hq < 1 || Hkv < 1 || D < 1 || 2 * (wq + wkv) > (1 << 30)) return ZGCM_ERR_INVALID_ARG;
    int st = check_widths(T, {d_model, (int)wq, (int)wkv});
    if (st == ZGCM_OK) st = check_ptrs({x, w_qkvg, dq, dk, dv, dg, dx, dw_qkvg});
    if (st != ZGCM_OK) return st;
    const void* parts[4] = {dq, dk, dv, dg};
    const int width[4] = {(int)wq, (int)wkv, (int)wkv, (int)wq};
    const int n_out = (int)(2 * (wq + wkv));
    // dx [T, d_model] = [dq|dk|dv|dg] W: A split along K, B = W as [K, N]
    GemmDesc a;
    a.M = T;
    a.N = d_model;
    a.K = n_out;
    a.a_split = 1;
    a.a_nseg = 4;
    // dW [n_out, d_model] = [dq|dk|dv|dg]^T x: A = the transpose of the parts, split along M
    GemmDesc w;
    w.M = n_out;
    w.N = d_model;
    w.K = T;
    w.a_mn = 1;
    w.a_split = 2;
    w.a_nseg = 4;
    int start = 0;
    for (int s = 0; s < 4; ++s) {
        a.a[s] = GemmSeg{parts[s], T, width[s], start};   // [T, width]: [M, K_part]
        w.a[s] = GemmSeg{parts[s], T, width[s], start};   // [T, width]: [K, M_part]
        start += width[s];
    }
    a.b_kn = 1;
    a.b = w_qkvg;
    a.c[0] = dx;
    a.c_ld[0] = d_model;
    w.b_kn = 1;
    w.b = x;
    w.c[0] = dw_qkvg;
    w.c_ld[0] = d_model;
    st = run(a, cuda_stream);
    return st == ZGCM_OK ? run(w, cuda_stream) : st;
}

int zgcm_proj_out_fwd(const void* a, const void* w_o, int T, int d_in, int d_model, void* y, void* cuda_stream) {
    int st = check_widths(T, {d_in, d_model});
    if (st == ZGCM_OK) st = check_ptrs({a, w_o, y});
    if (st != ZGCM_OK) return st;
    GemmDesc d;  // y [T, d_model] = a W_o^T: W_o is [N, K]
    d.M = T;
    d.N = d_model;
    d.K = d_in;
    d.a[0] = GemmSeg{a, T, d_in, 0};
    d.b = w_o;
    d.c[0] = y;
    d.c_ld[0] = d_model;
    return run(d, cuda_stream);
}

int zgcm_proj_out_bwd(const void* a, const void* w_o, const void* dy, int T, int d_in, int d_model, void* da,
                      void* dw_o, void* cuda_stream) {
    int st = check_widths(T, {d_in, d_model});
    if (st == ZGCM_OK) st = check_ptrs({a, w_o, dy, da, dw_o});
    if (st != ZGCM_OK) return st;
    GemmDesc x;  // da [T, d_in] = dy W_o: W_o is [K, N]
    x.M = T;
    x.N = d_in;
    x.K = d_model;
    x.a[0] = GemmSeg{dy, T, d_model, 0};
    x.b_kn = 1;
    x.b = w_o;
    x.c[0] = da;
    x.c_ld[0] = d_in;
    GemmDesc w;  // dW_o [d_model, d_in] = dy^T a: A is dy as [K, M], B = a as [K, N]
    w.M = d_model;
    w.N = d_in;
    w.K = T;
    w.a_mn = 1;
    w.a[0] = GemmSeg{dy, T, d_model, 0};
    w.b_kn = 1;
    w.b = a;
    w.c[0] = dw_o;
    w.c_ld[0] = d_in;
    st = run(x, cuda_stream);
    return st == ZGCM_OK ? run(w, cuda_stream) : st;
}

}  // extern "C"
