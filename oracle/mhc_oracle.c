/*
 * mhc_oracle.c -- fp64 CPU oracle for the mHC pre and post stages.
 *
 * TEST INFRASTRUCTURE ONLY (see mhc_oracle.h): used by the tests, the smoke
 * check and the benchmark's CPU-baseline leg; never by the product path.
 *
 * Every step follows the definitions on the pages in their order, with no
 * blocking, fusion or reordering: one token at a time, plain loops.  Tokens
 * are independent, so the optional OpenMP loop over tokens changes nothing in
 * the arithmetic of any token.
 */
#include "mhc_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Sinkhorn-Knopp: "DeepSeek-V4/mhc" page, equations sinkhorn-init and sinkhorn
 * (M0 = exp(B~), Mt = T_r(T_c(M(t-1)))); slavadubrov.com article, section
 * "Sinkhorn-Knopp-projectie" (columns first, then rows, 20 rounds). */
void oracle_sinkhorn(const double* logits, int n, int t_max, double* out)
{
    for (int k = 0; k < n * n; ++k) out[k] = exp(logits[k]);
    for (int it = 0; it < t_max; ++it) {
        /* T_c: divide every column by its sum */
        for (int j = 0; j < n; ++j) {
            double s = 0.0;
            for (int i = 0; i < n; ++i) s += out[i * n + j];
            for (int i = 0; i < n; ++i) out[i * n + j] = out[i * n + j] / s;
        }
        /* T_r: divide every row by its sum */
        for (int i = 0; i < n; ++i) {
            double s = 0.0;
            for (int j = 0; j < n; ++j) s += out[i * n + j];
            for (int j = 0; j < n; ++j) out[i * n + j] = out[i * n + j] / s;
        }
    }
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* One token of the pre stage.  work: [n*d + m + n*n] doubles of scratch. */
static void pre_one_token(const double* Xt, const double* phi,
                          const double* b_pre, const double* b_post, const double* b_res,
                          double alpha_pre, double alpha_post, double alpha_res,
                          int n, int d, double eps, int t_max,
                          double* x_in_t, double* H_t, double* work)
{
    const int nd = n * d;
    const int m = n * n + 2 * n;
    double* xhat = work;          /* [nd]  */
    double* h = xhat + nd;        /* [m]   */
    double* lres = h + m;         /* [n*n] */

    /* vec(X): row-stacked flatten, element (i, c) at index i*d + c.
     * RMSNorm over the n*d entries, eps inside the square root, no gain. */
    double ss = 0.0;
    for (int k = 0; k < nd; ++k) ss += Xt[k] * Xt[k];
    const double r = sqrt(ss / (double)nd + eps);
    for (int k = 0; k < nd; ++k) xhat[k] = Xt[k] / r;

    /* h = x_hat . phi, phi is [nd, m] row-major */
    for (int j = 0; j < m; ++j) h[j] = 0.0;
    for (int k = 0; k < nd; ++k)
        for (int j = 0; j < m; ++j) h[j] += xhat[k] * phi[(long)k * m + j];

    /* Logits (equations a/b/c-tilde) and the constrained maps. */
    for (int i = 0; i < n; ++i)
        H_t[i] = sigmoid(alpha_pre * h[i] + b_pre[i]);                       /* H_pre  */
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j)
            lres[i * n + j] = alpha_res * h[n + i * n + j] + b_res[i * n + j];
    oracle_sinkhorn(lres, n, t_max, H_t + n);                                /* H_res  */
    for (int i = 0; i < n; ++i)
        H_t[n + n * n + i] = 2.0 * sigmoid(alpha_post * h[n + n * n + i] + b_post[i]); /* H_post */

    /* Read map on the raw streams: x_in = sum_i H_pre[i] X[i, :] */
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += H_t[i] * Xt[i * d + c];
        x_in_t[c] = acc;
    }
}

int oracle_threads_used(int nthreads)
{
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = 1;
    int used = 1;
#pragma omp parallel num_threads(nthreads)
    {
#pragma omp single
        used = omp_get_num_threads();
    }
    return used;
#else
    (void)nthreads;
    return 1;
#endif
}

void oracle_mhc_pre(const double* X, const double* phi,
                    const double* b_pre, const double* b_post, const double* b_res,
                    double alpha_pre, double alpha_post, double alpha_res,
                    long T, int n, int d, double eps, int t_max,
                    double* x_in, double* H, int nthreads)
{
    const int nd = n * d;
    const int m = n * n + 2 * n;
    if (nthreads <= 0) nthreads = 1;
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* work = (double*)malloc(sizeof(double) * (size_t)(nd + m + n * n));
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
        for (long t = 0; t < T; ++t)
            pre_one_token(X + t * (long)nd, phi, b_pre, b_post, b_res,
                          alpha_pre, alpha_post, alpha_res, n, d, eps, t_max,
                          x_in + t * (long)d, H + t * (long)m, work);
        free(work);
    }
}

/* Post/res merge: slavadubrov.com article Eq. 3 and the knowledge page's HC
 * update; X'_i = sum_j H_res[i][j] X_j + H_post[i] F_out. */
void oracle_mhc_post(const double* X, const double* F_out, const double* H,
                     long T, int n, int d, double* X_out, int nthreads)
{
    const int m = n * n + 2 * n;
    if (nthreads <= 0) nthreads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (long t = 0; t < T; ++t) {
        const double* Xt = X + t * (long)n * d;
        const double* Ft = F_out + t * (long)d;
        const double* Hres = H + t * (long)m + n;
        const double* Hpost = H + t * (long)m + n + n * n;
        double* Ot = X_out + t * (long)n * d;
        for (int i = 0; i < n; ++i)
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int j = 0; j < n; ++j) acc += Hres[i * n + j] * Xt[j * d + c];
                Ot[i * d + c] = acc + Hpost[i] * Ft[c];
            }
    }
}
