/*
 * oracle_attention.c -- fp64 reference for exact softmax attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes is the plain, undecomposed definition that the
 * decomposition is claimed to reproduce exactly ("Stream-CQSA: Exact
 * Out-of-Memory Recovery for Attention", arXiv abstract: recomposition
 * recovers the full attention output; layerthelatestinalattice.com summary:
 * recomposition is mathematically equivalent to full-sequence attention).
 * For head h and query row i, over the allowed key set J(i) (all keys, or
 * keys j <= i when causal):
 *
 *     s_ij  = scale * <q_i, k_j>
 *     m_i   = max_{j in J(i)} s_ij
 *     lse_i = m_i + ln sum_{j in J(i)} exp(s_ij - m_i)
 *     o_i   = sum_{j in J(i)} exp(s_ij - lse_i) * v_j
 *
 * Everything is double precision.  Inputs are read in their stored type
 * (fp32, or bf16 given as raw 16-bit patterns) and widened exactly.
 * Layout: q, k, v are [N, H, d] row-major (one sequence).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_FP32 0
#define ORACLE_BF16 1

/* Exact widening of one stored element to double. */
static double load_elem(const void *base, int dtype, int64_t idx) {
    if (dtype == ORACLE_FP32) {
        return (double)((const float *)base)[idx];
    }
    /* bf16 is the upper half of an IEEE binary32 pattern. */
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * One (row, head) pair.  s is a caller-provided scratch of N doubles.
 * Writes d values to o and returns lse.
 */
static double attend_one(const void *q, const void *k, const void *v,
                         int dtype, int64_t N, int H, int d, int causal,
                         double scale, int64_t i, int h, double *s,
                         double *o) {
    const int64_t row_stride = (int64_t)H * d;
    const int64_t jmax = causal ? i + 1 : N;
    double m = -INFINITY;
    for (int64_t j = 0; j < jmax; ++j) {
        double dot = 0.0;
        for (int t = 0; t < d; ++t) {
            dot += load_elem(q, dtype, i * row_stride + (int64_t)h * d + t) *
                   load_elem(k, dtype, j * row_stride + (int64_t)h * d + t);
        }
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j < jmax; ++j) sum += exp(s[j] - m);
    const double lse = m + log(sum);
    for (int t = 0; t < d; ++t) o[t] = 0.0;
    for (int64_t j = 0; j < jmax; ++j) {
        const double w = exp(s[j] - lse);
        for (int t = 0; t < d; ++t)
            o[t] += w * load_elem(v, dtype, j * row_stride + (int64_t)h * d + t);
    }
    return lse;
}

/*
 * Attention for a chosen list of query rows (all heads each).
 *   rows   : nrows query indices in [0, N)
 *   out    : [nrows, H, d] doubles
 *   lse    : [nrows, H] doubles (natural log)
 * Returns 0 on success, -1 on bad arguments or allocation failure.
 */
int oracle_attention_rows(const void *q, const void *k, const void *v,
                          int dtype, int64_t N, int H, int d, int causal,
                          double scale, const int64_t *rows, int64_t nrows,
                          double *out, double *lse) {
    if (!q || !k || !v || !rows || !out || !lse) return -1;
    if (N <= 0 || H <= 0 || d <= 0 || nrows < 0) return -1;
    if (dtype != ORACLE_FP32 && dtype != ORACLE_BF16) return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return -1;
    int failed = 0;
    const int64_t work = nrows * (int64_t)H;
#pragma omp parallel
    {
        double *s = (double *)malloc((size_t)N * sizeof(double));
        if (!s) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t w = 0; w < work; ++w) {
                const int64_t r = w / H;
                const int h = (int)(w % H);
                double *o = out + (r * H + h) * (int64_t)d;
                lse[r * H + h] = attend_one(q, k, v, dtype, N, H, d, causal,
                                            scale, rows[r], h, s, o);
            }
            free(s);
        }
    }
    return failed ? -1 : 0;
}

/*
 * Full softmax weight matrix for tiny problems: probs [H, N, N], with
 * probs[h][i][j] = exp(s_ij - lse_i) for allowed j and 0 otherwise.
 * Used only to check that every row of weights sums to one.
 */
int oracle_attention_probs(const void *q, const void *k, int dtype, int64_t N,
                           int H, int d, int causal, double scale,
                           double *probs) {
    if (!q || !k || !probs || N <= 0 || H <= 0 || d <= 0) return -1;
    if (dtype != ORACLE_FP32 && dtype != ORACLE_BF16) return -1;
    const int64_t row_stride = (int64_t)H * d;
    for (int h = 0; h < H; ++h) {
        for (int64_t i = 0; i < N; ++i) {
            double *p = probs + ((int64_t)h * N + i) * N;
            const int64_t jmax = causal ? i + 1 : N;
            double m = -INFINITY;
            for (int64_t j = 0; j < N; ++j) p[j] = 0.0;
            for (int64_t j = 0; j < jmax; ++j) {
                double dot = 0.0;
                for (int t = 0; t < d; ++t)
                    dot += load_elem(q, dtype, i * row_stride + (int64_t)h * d + t) *
                           load_elem(k, dtype, j * row_stride + (int64_t)h * d + t);
                p[j] = scale * dot;
                if (p[j] > m) m = p[j];
            }
            double sum = 0.0;
            for (int64_t j = 0; j < jmax; ++j) sum += exp(p[j] - m);
            const double lse = m + log(sum);
            for (int64_t j = 0; j < jmax; ++j) p[j] = exp(p[j] - lse);
        }
    }
    return 0;
}

/*
 * Backward of the same definition.  With dO the gradient of the loss with
 * respect to the output (layout [N, H, d], the dtype of q, k, v):
 *
 *     D_i   = <dO_i, o_i>
 *     P_ij  = exp(s_ij - lse_i)                        for j in J(i)
 *     dP_ij = <dO_i, v_j>
 *     dS_ij = P_ij * (dP_ij - D_i)
 *     dq_i  = scale * sum_{j in J(i)} dS_ij k_j
 *     dk_j  = scale * sum_{i : j in J(i)} dS_ij q_i
 *     dv_j  = sum_{i : j in J(i)} P_ij dO_i
 *
 * (the chain rule through o_i = sum_j P_ij v_j and the softmax; the
 * decomposition recomputes P from the merged lse task by task, so each task
 * adds its allowed pairs' terms and the sums are exact).  Two plain passes,
 * so that no two threads write one gradient: dq by query row, dk and dv by
 * key row.
 */
static double dot_rows(const void *a, const void *b, int dtype, int64_t ia,
                       int64_t ib, int64_t row_stride, int h, int d) {
    double acc = 0.0;
    for (int t = 0; t < d; ++t)
        acc += load_elem(a, dtype, ia * row_stride + (int64_t)h * d + t) *
               load_elem(b, dtype, ib * row_stride + (int64_t)h * d + t);
    return acc;
}

/*
 * dq for chosen query rows (all heads).  dq, lse_out, D_out: [nrows, H, d]
 * and [nrows, H]; lse_out / D_out may be NULL.  Returns 0, or -1 on bad
 * arguments or allocation failure.
 */
int oracle_attention_backward_dq(const void *q, const void *k, const void *v,
                                 const void *dout, int dtype, int64_t N, int H,
                                 int d, int causal, double scale,
                                 const int64_t *rows, int64_t nrows,
                                 double *dq, double *lse_out, double *D_out) {
    if (!q || !k || !v || !dout || !rows || !dq) return -1;
    if (N <= 0 || H <= 0 || d <= 0 || nrows < 0) return -1;
    if (dtype != ORACLE_FP32 && dtype != ORACLE_BF16) return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return -1;
    const int64_t row_stride = (int64_t)H * d;
    int failed = 0;
    const int64_t work = nrows * (int64_t)H;
#pragma omp parallel
    {
        double *s = (double *)malloc((size_t)N * sizeof(double));
        double *o = (double *)malloc((size_t)d * sizeof(double));
        if (!s || !o) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t w = 0; w < work; ++w) {
                const int64_t r = w / H;
                const int h = (int)(w % H);
                const int64_t i = rows[r];
                const double lse = attend_one(q, k, v, dtype, N, H, d, causal,
                                              scale, i, h, s, o);
                double D = 0.0;
                for (int t = 0; t < d; ++t)
                    D += load_elem(dout, dtype, i * row_stride + (int64_t)h * d + t) * o[t];
                double *g = dq + (r * H + h) * (int64_t)d;
                for (int t = 0; t < d; ++t) g[t] = 0.0;
                const int64_t jmax = causal ? i + 1 : N;
                for (int64_t j = 0; j < jmax; ++j) {
                    const double P = exp(s[j] - lse);
                    const double dP = dot_rows(dout, v, dtype, i, j, row_stride, h, d);
                    const double dS = P * (dP - D);
                    for (int t = 0; t < d; ++t)
                        g[t] += scale * dS * load_elem(k, dtype, j * row_stride + (int64_t)h * d + t);
                }
                if (lse_out) lse_out[r * H + h] = lse;
                if (D_out) D_out[r * H + h] = D;
            }
        }
        free(s);
        free(o);
    }
    return failed ? -1 : 0;
}

/*
 * dk and dv for chosen key rows (all heads): [nkeys, H, d] each.  Needs
 * lse_i and D_i of every query row first (O(N^2 H d)).
 */
int oracle_attention_backward_dkdv(const void *q, const void *k, const void *v,
                                   const void *dout, int dtype, int64_t N, int H,
                                   int d, int causal, double scale,
                                   const int64_t *keys, int64_t nkeys,
                                   double *dk, double *dv) {
    if (!q || !k || !v || !dout || !keys || !dk || !dv) return -1;
    if (N <= 0 || H <= 0 || d <= 0 || nkeys < 0) return -1;
    if (dtype != ORACLE_FP32 && dtype != ORACLE_BF16) return -1;
    for (int64_t r = 0; r < nkeys; ++r)
        if (keys[r] < 0 || keys[r] >= N) return -1;
    const int64_t row_stride = (int64_t)H * d;
    double *lse = (double *)malloc((size_t)N * H * sizeof(double));
    double *Dv = (double *)malloc((size_t)N * H * sizeof(double));
    if (!lse || !Dv) {
        free(lse);
        free(Dv);
        return -1;
    }
    int failed = 0;
    const int64_t work = N * (int64_t)H;
#pragma omp parallel
    {
        double *s = (double *)malloc((size_t)N * sizeof(double));
        double *o = (double *)malloc((size_t)d * sizeof(double));
        if (!s || !o) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t w = 0; w < work; ++w) {
                const int64_t i = w / H;
                const int h = (int)(w % H);
                lse[w] = attend_one(q, k, v, dtype, N, H, d, causal, scale, i, h, s, o);
                double D = 0.0;
                for (int t = 0; t < d; ++t)
                    D += load_elem(dout, dtype, i * row_stride + (int64_t)h * d + t) * o[t];
                Dv[w] = D;
            }
        }
        free(s);
        free(o);
    }
    if (!failed) {
        const int64_t kwork = nkeys * (int64_t)H;
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t w = 0; w < kwork; ++w) {
            const int64_t r = w / H;
            const int h = (int)(w % H);
            const int64_t j = keys[r];
            double *gk = dk + (r * H + h) * (int64_t)d;
            double *gv = dv + (r * H + h) * (int64_t)d;
            for (int t = 0; t < d; ++t) gk[t] = gv[t] = 0.0;
            for (int64_t i = causal ? j : 0; i < N; ++i) {
                const double sij = scale * dot_rows(q, k, dtype, i, j, row_stride, h, d);
                const double P = exp(sij - lse[i * H + h]);
                const double dP = dot_rows(dout, v, dtype, i, j, row_stride, h, d);
                const double dS = P * (dP - Dv[i * H + h]);
                for (int t = 0; t < d; ++t) {
                    const int64_t ix = i * row_stride + (int64_t)h * d + t;
                    gk[t] += scale * dS * load_elem(q, dtype, ix);
                    gv[t] += P * load_elem(dout, dtype, ix);
                }
            }
        }
    }
    free(lse);
    free(Dv);
    return failed ? -1 : 0;
}

/* Number of OpenMP threads a parallel region of this library will use. */
int oracle_num_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
