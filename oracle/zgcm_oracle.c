/*
 * zgcm_oracle.c — plain fp64 CPU oracle of the ZGCM-1 gated window-attention layer.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load this library.  It shares no code with the GPU path: it has its
 * own normalisation, rotation, softmax, gate and gradient arithmetic, written as the plain
 * definitions in double precision, with no blocking, fusion or reordering.
 *
 * What it computes (the layer as the ZGCM-1 pages describe it):
 *   - QK-RMSNorm and partial RoPE (ratio 0.33 -> 42 of 128 dims), GQA with 32 query heads
 *     over 8 KV heads: shibing624 review, section "架构：5:1 的门控滑窗注意力"; ZGCM-1
 *     summary (paper.rainbus.top), section "核心方法".
 *   - causal attention over the 128 nearest keys; global layers = the same with the window
 *     at least the sequence length: ZGCM-1 summary, section "前置知识 / 滑动窗口注意力
 *     (SWA)与混合注意力".
 *   - the sigmoid output gate: shibing624 review, section "架构" (formula lost from the page;
 *     read as out = sigmoid(g) * attn, elementwise).
 * Readings where the pages are silent (each listed in the design notes): key j is visible
 * to query i iff i-W < j <= i; RMSNorm r = sqrt(mean_d x^2 + eps), y = gamma * x / r; norm
 * before rotation; rotation pairs (t, t+R/2) with theta_t = base^(-2t/R) and positions
 * 0..S-1; query head h reads KV head h / (Hq/Hkv); lse in natural log of the scaled scores.
 *
 * Backward: exact gradients of L = sum(dout * out) w.r.t. q, k, v, g, gamma_q, gamma_k by
 * the chain rule through the same definitions (softmax, rotation transpose, RMSNorm).
 *
 * Inputs are double arrays: the caller upcasts the bf16 tensors exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double* q;       /* [B,S,Hq,D]  */
    const double* k;       /* [B,S,Hkv,D] */
    const double* v;       /* [B,S,Hkv,D] */
    const double* g;       /* [B,S,Hq,D]  gate logits */
    const double* gamma_q; /* [D] */
    const double* gamma_k; /* [D] */
    int64_t B, S, Hq, Hkv, D, R, W;
    double base, eps, scale;
} zo_problem;

/* ---------- indexing ---------- */

static const double* qrow(const zo_problem* P, int64_t b, int64_t s, int64_t h) {
    return P->q + ((b * P->S + s) * P->Hq + h) * P->D;
}
static const double* grow(const zo_problem* P, int64_t b, int64_t s, int64_t h) {
    return P->g + ((b * P->S + s) * P->Hq + h) * P->D;
}
static const double* krow(const zo_problem* P, int64_t b, int64_t s, int64_t h) {
    return P->k + ((b * P->S + s) * P->Hkv + h) * P->D;
}
static const double* vrow(const zo_problem* P, int64_t b, int64_t s, int64_t h) {
    return P->v + ((b * P->S + s) * P->Hkv + h) * P->D;
}
static int64_t kv_head_of(const zo_problem* P, int64_t h) { return h / (P->Hq / P->Hkv); }

/* first visible key of query i: key j visible iff i - W < j <= i */
static int64_t window_lo(const zo_problem* P, int64_t i) {
    int64_t lo = i - P->W + 1;
    return lo < 0 ? 0 : lo;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ---------- QK-RMSNorm followed by partial RoPE ---------- */

/* rotation angle of pair t at position pos */
static double rope_angle(const zo_problem* P, int64_t t, int64_t pos) {
    double theta = pow(P->base, -2.0 * (double)t / (double)P->R);
    return (double)pos * theta;
}

/*
 * y = RoPE(gamma * x / r),  r = sqrt(mean_d x^2 + eps).
 * Writes the rotated row to y; xhat (= x / r) and r if requested.
 */
static void zo_prologue(const zo_problem* P, const double* x, const double* gamma, int64_t pos,
                        double* y, double* xhat, double* r_out) {
    const int64_t D = P->D, half = P->R / 2;
    double ss = 0.0;
    for (int64_t d = 0; d < D; ++d) ss += x[d] * x[d];
    const double r = sqrt(ss / (double)D + P->eps);
    for (int64_t d = 0; d < D; ++d) {
        double xh = x[d] / r;
        if (xhat) xhat[d] = xh;
        y[d] = gamma[d] * xh;
    }
    for (int64_t t = 0; t < half; ++t) {
        double a = rope_angle(P, t, pos), c = cos(a), s = sin(a);
        double y1 = y[t], y2 = y[t + half];
        y[t] = y1 * c - y2 * s;
        y[t + half] = y2 * c + y1 * s;
    }
    if (r_out) *r_out = r;
}

/*
 * Given dL/dy_rot for y_rot = RoPE(gamma * x / r), returns dL/dx and adds dL/dgamma.
 *   dy     = R^T dy_rot                       (transpose of the pair rotation)
 *   dgamma += dy * xhat
 *   dxhat  = dy * gamma
 *   dx     = (dxhat - xhat * mean_d(dxhat * xhat)) / r
 */
static void zo_prologue_backward(const zo_problem* P, const double* x, const double* gamma,
                                 int64_t pos, const double* dyrot, double* dx, double* dgamma,
                                 double* scratch /* 2*D */) {
    const int64_t D = P->D, half = P->R / 2;
    double* xhat = scratch;
    double* dy = scratch + D;
    double ss = 0.0;
    for (int64_t d = 0; d < D; ++d) ss += x[d] * x[d];
    const double r = sqrt(ss / (double)D + P->eps);
    for (int64_t d = 0; d < D; ++d) {
        xhat[d] = x[d] / r;
        dy[d] = dyrot[d];
    }
    for (int64_t t = 0; t < half; ++t) {
        double a = rope_angle(P, t, pos), c = cos(a), s = sin(a);
        double d1 = dyrot[t], d2 = dyrot[t + half];
        dy[t] = d1 * c + d2 * s;
        dy[t + half] = -d1 * s + d2 * c;
    }
    double m = 0.0;
    for (int64_t d = 0; d < D; ++d) {
        if (dgamma) dgamma[d] += dy[d] * xhat[d];
        m += dy[d] * gamma[d] * xhat[d];
    }
    m /= (double)D;
    for (int64_t d = 0; d < D; ++d) dx[d] = (dy[d] * gamma[d] - xhat[d] * m) / r;
}

/* ---------- k_hat table: rows are computed only where `need` is set ---------- */

static double* khat_table(const zo_problem* P, const unsigned char* need) {
    const int64_t nrows = P->B * P->S * P->Hkv;
    double* kh = (double*)malloc((size_t)(nrows > 0 ? nrows : 1) * (size_t)P->D * sizeof(double));
    if (!kh) return NULL;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < nrows; ++row) {
        if (need && !need[row / P->Hkv]) continue; /* need is per (b, s) */
        int64_t bs = row / P->Hkv, h = row % P->Hkv;
        int64_t b = bs / P->S, s = bs % P->S;
        zo_prologue(P, krow(P, b, s, h), P->gamma_k, s, kh + row * P->D, NULL, NULL);
    }
    return kh;
}

static const double* khat_row(const zo_problem* P, const double* kh, int64_t b, int64_t s, int64_t h) {
    return kh + ((b * P->S + s) * P->Hkv + h) * P->D;
}

/* ---------- one query row ---------- */

/*
 * Attention of query (b, i, h) with its rotated, normalised q_hat.
 * p[0 .. n) receives softmax probabilities of keys lo .. i (n = i - lo + 1),
 * A receives sum_j p_j v_j, *lse the natural-log normaliser of the scaled scores.
 */
static void zo_attend_row(const zo_problem* P, const double* kh, int64_t b, int64_t i, int64_t h,
                          const double* qhat, double* p, double* A, double* lse) {
    const int64_t D = P->D, kvh = kv_head_of(P, h), lo = window_lo(P, i), n = i - lo + 1;
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
        const double* kj = khat_row(P, kh, b, lo + t, kvh);
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qhat[d] * kj[d];
        p[t] = P->scale * dot;
        if (p[t] > m) m = p[t];
    }
    double l = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        p[t] = exp(p[t] - m);
        l += p[t];
    }
    for (int64_t t = 0; t < n; ++t) p[t] /= l;
    for (int64_t d = 0; d < D; ++d) A[d] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        const double* vj = vrow(P, b, lo + t, kvh);
        for (int64_t d = 0; d < D; ++d) A[d] += p[t] * vj[d];
    }
    *lse = m + log(l);
}

/*
 * Backward of query row (b, i, h), given its probabilities p and pre-gate output A.
 *   dA = dout * sigmoid(g);  dg = dout * A * sigmoid(g) * (1 - sigmoid(g))
 *   dp_j = dA . v_j;  Delta = sum_j p_j dp_j;  ds_j = p_j (dp_j - Delta)
 *   dq_hat = scale * sum_j ds_j k_hat_j
 * ds (length n) and dA are returned for key-side accumulation.
 */
static void zo_row_backward(const zo_problem* P, const double* kh, int64_t b, int64_t i, int64_t h,
                            const double* dout_row, const double* p, const double* A,
                            double* dA, double* dg_row, double* ds, double* dqhat) {
    const int64_t D = P->D, kvh = kv_head_of(P, h), lo = window_lo(P, i), n = i - lo + 1;
    const double* gr = grow(P, b, i, h);
    for (int64_t d = 0; d < D; ++d) {
        double sg = sigmoid(gr[d]);
        dA[d] = dout_row[d] * sg;
        if (dg_row) dg_row[d] = dout_row[d] * A[d] * sg * (1.0 - sg);
    }
    double delta = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        const double* vj = vrow(P, b, lo + t, kvh);
        double dp = 0.0;
        for (int64_t d = 0; d < D; ++d) dp += dA[d] * vj[d];
        ds[t] = dp;
        delta += p[t] * dp;
    }
    for (int64_t t = 0; t < n; ++t) ds[t] = p[t] * (ds[t] - delta);
    if (dqhat) {
        for (int64_t d = 0; d < D; ++d) dqhat[d] = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            const double* kj = khat_row(P, kh, b, lo + t, kvh);
            for (int64_t d = 0; d < D; ++d) dqhat[d] += P->scale * ds[t] * kj[d];
        }
    }
}

static int zo_check(const zo_problem* P) {
    if (P->B < 0 || P->S < 0 || P->Hq < 1 || P->Hkv < 1 || P->D < 1) return -1;
    if (P->Hq % P->Hkv != 0) return -1;
    if (P->R < 0 || P->R > P->D || (P->R % 2) != 0) return -1;
    if (P->W < 1) return -1;
    return 0;
}

/* mark the (b, s) rows whose k_hat the listed query rows read */
static unsigned char* need_for_queries(const zo_problem* P, const int64_t* rows, int64_t nrows) {
    unsigned char* need = (unsigned char*)calloc((size_t)(P->B * P->S > 0 ? P->B * P->S : 1), 1);
    if (!need) return NULL;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t bs = rows ? rows[r] : r, b = bs / P->S, i = bs % P->S;
        for (int64_t j = window_lo(P, i); j <= i; ++j) need[b * P->S + j] = 1;
    }
    return need;
}

/* ============================ exported entry points ============================ */

/* Normalised, rotated row (exposed so the rotation can be pinned on its own). */
void zo_prologue_row(const zo_problem* P, const double* x, const double* gamma, int64_t pos,
                     double* y) {
    zo_prologue(P, x, gamma, pos, y, NULL, NULL);
}

/*
 * Forward of the listed query rows (flattened b*S + i), all query heads, or of every row
 * when rows == NULL (then nrows must be B*S).
 * out [nrows, Hq, D], lse [nrows, Hq].
 */
int zo_forward(const zo_problem* P, const int64_t* rows, int64_t nrows, double* out, double* lse) {
    if (zo_check(P)) return -1;
    if (nrows == 0) return 0;
    unsigned char* need = need_for_queries(P, rows, nrows);
    double* kh = need ? khat_table(P, need) : NULL;
    if (!kh) { free(need); return -2; }
    const int64_t D = P->D, Hq = P->Hq;
    int rc = 0;
#pragma omp parallel
    {
        double* qh = (double*)malloc(sizeof(double) * (size_t)D);
        double* A = (double*)malloc(sizeof(double) * (size_t)D);
        int64_t pmax = P->W < P->S ? P->W : P->S;
        double* p = (double*)malloc(sizeof(double) * (size_t)(pmax > 0 ? pmax : 1));
        if (!qh || !A || !p) {
#pragma omp atomic write
            rc = -2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < nrows * Hq; ++t) {
                int64_t r = t / Hq, h = t % Hq;
                int64_t bs = rows ? rows[r] : r, b = bs / P->S, i = bs % P->S;
                zo_prologue(P, qrow(P, b, i, h), P->gamma_q, i, qh, NULL, NULL);
                double l;
                zo_attend_row(P, kh, b, i, h, qh, p, A, &l);
                const double* gr = grow(P, b, i, h);
                double* o = out + (r * Hq + h) * D;
                for (int64_t d = 0; d < D; ++d) o[d] = sigmoid(gr[d]) * A[d];
                lse[r * Hq + h] = l;
            }
        }
        free(qh); free(A); free(p);
    }
    free(kh); free(need);
    return rc;
}

/*
 * Backward, query side, for the listed query rows (or all rows when rows == NULL):
 * dq [nrows, Hq, D] (gradient w.r.t. raw q) and dg [nrows, Hq, D].
 */
int zo_backward_qrows(const zo_problem* P, const double* dout, const int64_t* rows, int64_t nrows,
                      double* dq, double* dg) {
    if (zo_check(P)) return -1;
    if (nrows == 0) return 0;
    unsigned char* need = need_for_queries(P, rows, nrows);
    double* kh = need ? khat_table(P, need) : NULL;
    if (!kh) { free(need); return -2; }
    const int64_t D = P->D, Hq = P->Hq;
    int rc = 0;
#pragma omp parallel
    {
        int64_t pmax = P->W < P->S ? P->W : P->S;
        if (pmax < 1) pmax = 1;
        double* buf = (double*)malloc(sizeof(double) * (size_t)(7 * D + 2 * pmax));
        if (!buf) {
#pragma omp atomic write
            rc = -2;
        } else {
            double *qh = buf, *A = buf + D, *dA = buf + 2 * D, *dqh = buf + 3 * D,
                   *scr = buf + 4 * D, *p = buf + 7 * D, *ds = buf + 7 * D + pmax;
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < nrows * Hq; ++t) {
                int64_t r = t / Hq, h = t % Hq;
                int64_t bs = rows ? rows[r] : r, b = bs / P->S, i = bs % P->S;
                const double* x = qrow(P, b, i, h);
                zo_prologue(P, x, P->gamma_q, i, qh, NULL, NULL);
                double l;
                zo_attend_row(P, kh, b, i, h, qh, p, A, &l);
                const double* dor = dout + ((b * P->S + i) * Hq + h) * D;
                zo_row_backward(P, kh, b, i, h, dor, p, A, dA, dg + (r * Hq + h) * D, ds, dqh);
                zo_prologue_backward(P, x, P->gamma_q, i, dqh, dq + (r * Hq + h) * D, NULL, scr);
            }
        }
        free(buf);
    }
    free(kh); free(need);
    return rc;
}

/*
 * Backward, key side, for the listed key rows (flattened b*S + j; NULL = all rows):
 * dk, dv [nrows, Hkv, D], both summed over the query heads that share the KV head.
 * Every query row whose window holds a listed key is processed once per (b, KV head).
 */
int zo_backward_krows(const zo_problem* P, const double* dout, const int64_t* rows, int64_t nrows,
                      double* dk, double* dv) {
    if (zo_check(P)) return -1;
    if (nrows == 0) return 0;
    const int64_t D = P->D, Hq = P->Hq, Hkv = P->Hkv, G = Hq / Hkv, S = P->S, B = P->B;
    /* slot[b*S + j] = index into rows of key row (b, j), or -1 */
    int64_t* slot = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B * S));
    unsigned char* qneed = (unsigned char*)calloc((size_t)(B * S), 1);
    unsigned char* kneed = (unsigned char*)calloc((size_t)(B * S), 1);
    if (!slot || !qneed || !kneed) { free(slot); free(qneed); free(kneed); return -2; }
    for (int64_t t = 0; t < B * S; ++t) slot[t] = -1;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t bs = rows ? rows[r] : r, b = bs / S, j = bs % S;
        slot[bs] = r;
        int64_t hi = j + P->W - 1 < S - 1 ? j + P->W - 1 : S - 1;
        for (int64_t i = j; i <= hi; ++i) qneed[b * S + i] = 1;
    }
    for (int64_t bs = 0; bs < B * S; ++bs)
        if (qneed[bs]) {
            int64_t b = bs / S, i = bs % S;
            for (int64_t j = window_lo(P, i); j <= i; ++j) kneed[b * S + j] = 1;
        }
    double* kh = khat_table(P, kneed);
    double* dkh = (double*)calloc((size_t)nrows * (size_t)(Hkv * D), sizeof(double));
    if (!kh || !dkh) { free(slot); free(qneed); free(kneed); free(kh); free(dkh); return -2; }
    for (int64_t t = 0; t < nrows * Hkv * D; ++t) dv[t] = 0.0;
    int rc = 0;
    /* one task per (b, KV head): it alone writes that head's slots, so sums are ordered */
#pragma omp parallel
    {
        int64_t pmax = P->W < S ? P->W : S;
        if (pmax < 1) pmax = 1;
        double* buf = (double*)malloc(sizeof(double) * (size_t)(4 * D + 2 * pmax));
        if (!buf) {
#pragma omp atomic write
            rc = -2;
        } else {
            double *qh = buf, *A = buf + D, *dA = buf + 2 * D, *scr = buf + 3 * D,
                   *p = buf + 4 * D, *ds = buf + 4 * D + pmax;
            (void)scr;
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < B * Hkv; ++task) {
                int64_t b = task / Hkv, kvh = task % Hkv;
                for (int64_t i = 0; i < S; ++i) {
                    if (!qneed[b * S + i]) continue;
                    for (int64_t h = kvh * G; h < (kvh + 1) * G; ++h) {
                        zo_prologue(P, qrow(P, b, i, h), P->gamma_q, i, qh, NULL, NULL);
                        double l;
                        zo_attend_row(P, kh, b, i, h, qh, p, A, &l);
                        const double* dor = dout + ((b * S + i) * Hq + h) * D;
                        zo_row_backward(P, kh, b, i, h, dor, p, A, dA, NULL, ds, NULL);
                        int64_t lo = window_lo(P, i);
                        for (int64_t j = lo; j <= i; ++j) {
                            int64_t r = slot[b * S + j];
                            if (r < 0) continue;
                            double pj = p[j - lo], dsj = ds[j - lo];
                            double* dvr = dv + (r * Hkv + kvh) * D;
                            double* dkr = dkh + (r * Hkv + kvh) * D;
                            for (int64_t d = 0; d < D; ++d) {
                                dvr[d] += pj * dA[d];
                                dkr[d] += P->scale * dsj * qh[d];
                            }
                        }
                    }
                }
            }
        }
        free(buf);
    }
    if (rc == 0) {
#pragma omp parallel
        {
            double* scr = (double*)malloc(sizeof(double) * (size_t)(2 * D));
#pragma omp for schedule(static)
            for (int64_t t = 0; t < nrows * Hkv; ++t) {
                int64_t r = t / Hkv, kvh = t % Hkv;
                int64_t bs = rows ? rows[r] : r, b = bs / S, j = bs % S;
                zo_prologue_backward(P, krow(P, b, j, kvh), P->gamma_k, j, dkh + t * D, dk + t * D,
                                     NULL, scr);
            }
            free(scr);
        }
    }
    free(slot); free(qneed); free(kneed); free(kh); free(dkh);
    return rc;
}

/*
 * Full backward: dq, dg [B,S,Hq,D]; dk, dv [B,S,Hkv,D]; dgamma_q, dgamma_k [D].
 * One task per (b, KV head) holds that head's key-side sums; d_gamma partials are kept
 * per task and added in task order, so the result does not depend on the thread count.
 */
int zo_backward_full(const zo_problem* P, const double* dout, double* dq, double* dk, double* dv,
                     double* dg, double* dgamma_q, double* dgamma_k) {
    if (zo_check(P)) return -1;
    const int64_t D = P->D, Hq = P->Hq, Hkv = P->Hkv, G = Hq / Hkv, S = P->S, B = P->B;
    for (int64_t d = 0; d < D; ++d) dgamma_q[d] = dgamma_k[d] = 0.0;
    if (B == 0 || S == 0) return 0;
    double* kh = khat_table(P, NULL);
    double* part = (double*)calloc((size_t)(B * Hkv) * (size_t)(2 * D), sizeof(double));
    if (!kh || !part) { free(kh); free(part); return -2; }
    int rc = 0;
#pragma omp parallel
    {
        int64_t pmax = P->W < S ? P->W : S;
        double* buf = (double*)malloc(sizeof(double) * (size_t)(7 * D + 2 * pmax));
        double* dkh = (double*)malloc(sizeof(double) * (size_t)(S * D));
        double* dvh = (double*)malloc(sizeof(double) * (size_t)(S * D));
        if (!buf || !dkh || !dvh) {
#pragma omp atomic write
            rc = -2;
        } else {
            double *qh = buf, *A = buf + D, *dA = buf + 2 * D, *dqh = buf + 3 * D,
                   *scr = buf + 4 * D, *dxk = buf + 6 * D, *p = buf + 7 * D, *ds = buf + 7 * D + pmax;
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < B * Hkv; ++task) {
                int64_t b = task / Hkv, kvh = task % Hkv;
                double* dgq = part + task * 2 * D;
                double* dgk = dgq + D;
                memset(dkh, 0, sizeof(double) * (size_t)(S * D));
                memset(dvh, 0, sizeof(double) * (size_t)(S * D));
                for (int64_t h = kvh * G; h < (kvh + 1) * G; ++h) {
                    for (int64_t i = 0; i < S; ++i) {
                        const double* x = qrow(P, b, i, h);
                        zo_prologue(P, x, P->gamma_q, i, qh, NULL, NULL);
                        double l;
                        zo_attend_row(P, kh, b, i, h, qh, p, A, &l);
                        const int64_t off = ((b * S + i) * Hq + h) * D;
                        zo_row_backward(P, kh, b, i, h, dout + off, p, A, dA, dg + off, ds, dqh);
                        zo_prologue_backward(P, x, P->gamma_q, i, dqh, dq + off, dgq, scr);
                        int64_t lo = window_lo(P, i);
                        for (int64_t j = lo; j <= i; ++j) {
                            double pj = p[j - lo], dsj = ds[j - lo];
                            for (int64_t d = 0; d < D; ++d) {
                                dvh[j * D + d] += pj * dA[d];
                                dkh[j * D + d] += P->scale * dsj * qh[d];
                            }
                        }
                    }
                }
                for (int64_t j = 0; j < S; ++j) {
                    const int64_t off = ((b * S + j) * Hkv + kvh) * D;
                    zo_prologue_backward(P, krow(P, b, j, kvh), P->gamma_k, j, dkh + j * D, dxk, dgk, scr);
                    for (int64_t d = 0; d < D; ++d) {
                        dk[off + d] = dxk[d];
                        dv[off + d] = dvh[j * D + d];
                    }
                }
            }
        }
        free(buf); free(dkh); free(dvh);
    }
    if (rc == 0)
        for (int64_t task = 0; task < B * Hkv; ++task)
            for (int64_t d = 0; d < D; ++d) {
                dgamma_q[d] += part[task * 2 * D + d];
                dgamma_k[d] += part[task * 2 * D + D + d];
            }
    free(kh); free(part);
    return rc;
}

/* threads the OpenMP runtime will use (reported beside the CPU baseline) */
#ifdef _OPENMP
#include <omp.h>
int zo_num_threads(void) { return omp_get_max_threads(); }
#else
int zo_num_threads(void) { return 1; }
#endif
