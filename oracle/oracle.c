/*
 * oracle.c — plain fp64 CPU reference for the low-rank linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the bench's CPU
 * baseline use it.  It shares no code with the CUDA library.
 *
 * What it computes (the plain definition, no blocking or reordering):
 *
 *   T[m,j] = sum_k X[m,k] * A[k,j]                 (j < r)
 *   Y[m,n] = sum_j T[m,j] * B[j,n]  + bias[n]      (n < N)
 *
 * This is the factorised layer that replaces a dense Y = X*W with W ~ A*B
 * ("Why Smaller Is Slower? Dimensional Misalignment in Compressed LLMs",
 * §1 Introduction, Figure 1: low-rank factorisation puts the reduced rank r
 * as the inner dimension of two smaller GEMMs; LowRankArena review,
 * "What SVD-based LLM compression actually does": the forward pass becomes
 * two small multiplies with k(m+n) stored parameters).  The pages write it
 * column-wise (y = A(Bx)); with row vectors (Y = X*W, X [M,K], W [K,N]) the
 * same product reads Y = (X*A)*B with A [K,r] and B [r,N].
 *
 * All arithmetic is IEEE fp64 on the exact widened bf16 inputs; T is not
 * rounded, Y is not rounded.  The bias is added after the sum over j.
 * Rows m are independent, so OpenMP splits the loop over m; within a row
 * the loops run in the plain order k then j, and j then n.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef void (*row_fetch)(const void *base, int64_t row, int64_t len,
                          int64_t ld, double *out);

static double bf16_value(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void fetch_bf16(const void *base, int64_t row, int64_t len, int64_t ld,
                       double *out) {
    const uint16_t *p = (const uint16_t *)base + row * ld;
    for (int64_t i = 0; i < len; ++i) out[i] = bf16_value(p[i]);
}

static void fetch_f64(const void *base, int64_t row, int64_t len, int64_t ld,
                      double *out) {
    const double *p = (const double *)base + row * ld;
    for (int64_t i = 0; i < len; ++i) out[i] = p[i];
}

/* One output row m: T row, then Y row.  Scratch: x[K], a[r], t[r], b[N]. */
static void one_row(row_fetch f, const void *X, const void *A, const void *B,
                    const void *bias, double *Yrow, int64_t m, int64_t K,
                    int64_t r, int64_t N, double *x, double *a, double *t,
                    double *b) {
    f(X, m, K, K, x);
    for (int64_t j = 0; j < r; ++j) t[j] = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        const double xk = x[k];
        f(A, k, r, r, a);
        for (int64_t j = 0; j < r; ++j) t[j] += xk * a[j];
    }
    for (int64_t n = 0; n < N; ++n) Yrow[n] = 0.0;
    for (int64_t j = 0; j < r; ++j) {
        const double tj = t[j];
        f(B, j, N, N, b);
        for (int64_t n = 0; n < N; ++n) Yrow[n] += tj * b[n];
    }
    if (bias) {
        f(bias, 0, N, N, b);
        for (int64_t n = 0; n < N; ++n) Yrow[n] += b[n];
    }
}

static int run_rows(row_fetch f, const void *X, const void *A, const void *B,
                    const void *bias, double *Y, int64_t K, int64_t r,
                    int64_t N, const int64_t *rows, int64_t n_rows,
                    int nthreads) {
    if (K < 0 || r < 0 || N < 0 || n_rows < 0) return 1;
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1) reduction(| : failed)
#endif
    {
        int64_t big = K > N ? K : N;
        double *x = (double *)malloc(sizeof(double) * (size_t)(K + 1));
        double *a = (double *)malloc(sizeof(double) * (size_t)(r + 1));
        double *t = (double *)malloc(sizeof(double) * (size_t)(r + 1));
        double *b = (double *)malloc(sizeof(double) * (size_t)(big + 1));
        if (!x || !a || !t || !b) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
            for (int64_t i = 0; i < n_rows; ++i) {
                one_row(f, X, A, B, bias, Y + i * N, rows[i], K, r, N, x, a,
                        t, b);
            }
        }
        free(x); free(a); free(t); free(b);
    }
    (void)nthreads;
    return failed;
}

static int64_t *all_rows(int64_t M) {
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(M + 1));
    if (rows)
        for (int64_t m = 0; m < M; ++m) rows[m] = m;
    return rows;
}

/* Y [M,N] fp64 from bf16 X [M,K], A [K,r], B [r,N], bias [N] (nullable). */
int oracle_lr_linear(const uint16_t *X, const uint16_t *A, const uint16_t *B,
                     const uint16_t *bias, double *Y, int64_t M, int64_t K,
                     int64_t r, int64_t N, int nthreads) {
    if (M < 0) return 1;
    int64_t *rows = all_rows(M);
    if (!rows) return 1;
    int rc = run_rows(fetch_bf16, X, A, B, bias, Y, K, r, N, rows, M, nthreads);
    free(rows);
    return rc;
}

/* Only the listed rows of X: Y has n_rows rows, Y[i] is output row rows[i]. */
int oracle_lr_linear_rows(const uint16_t *X, const uint16_t *A,
                          const uint16_t *B, const uint16_t *bias, double *Y,
                          int64_t K, int64_t r, int64_t N, const int64_t *rows,
                          int64_t n_rows, int nthreads) {
    return run_rows(fetch_bf16, X, A, B, bias, Y, K, r, N, rows, n_rows,
                    nthreads);
}

/* The same definition on fp64 inputs (used to pin the oracle against an exact
 * SVD, whose factors are not bf16 values). */
int oracle_lr_linear_f64(const double *X, const double *A, const double *B,
                         const double *bias, double *Y, int64_t M, int64_t K,
                         int64_t r, int64_t N, int nthreads) {
    if (M < 0) return 1;
    int64_t *rows = all_rows(M);
    if (!rows) return 1;
    int rc = run_rows(fetch_f64, X, A, B, bias, Y, K, r, N, rows, M, nthreads);
    free(rows);
    return rc;
}

/* Dense comparison Y = X*W + bias, W [K,N] (the layer before factorisation,
 * same paper, Figure 1).  Listed rows only, as above. */
int oracle_dense_rows(const uint16_t *X, const uint16_t *W,
                      const uint16_t *bias, double *Y, int64_t K, int64_t N,
                      const int64_t *rows, int64_t n_rows, int nthreads) {
    if (K < 0 || N < 0 || n_rows < 0) return 1;
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1) reduction(| : failed)
#endif
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)(K + 1));
        double *w = (double *)malloc(sizeof(double) * (size_t)(N + 1));
        if (!x || !w) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
            for (int64_t i = 0; i < n_rows; ++i) {
                double *y = Y + i * N;
                fetch_bf16(X, rows[i], K, K, x);
                for (int64_t n = 0; n < N; ++n) y[n] = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    const double xk = x[k];
                    fetch_bf16(W, k, N, N, w);
                    for (int64_t n = 0; n < N; ++n) y[n] += xk * w[n];
                }
                if (bias) {
                    fetch_bf16(bias, 0, N, N, w);
                    for (int64_t n = 0; n < N; ++n) y[n] += w[n];
                }
            }
        }
        free(x); free(w);
    }
    (void)nthreads;
    return failed;
}
