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

/* One token of the HC pre stage, the unconstrained comparison the mHC pages start from
 * (slavadubrov.com article, section "Kernmechanismen": in HC each map is a learned static
 * part, a bias, plus an input-dependent term passed through tanh, so its entries may take
 * either sign; the same article's "Details van de parameterisatie" names tanh as what mHC
 * replaces by the sigmoid).  The input-dependent term is read as the same normalised
 * projection h = RMSNorm(vec X) . phi that mHC uses, scaled by the map's alpha:
 *   H_pre = b_pre + alpha_pre tanh(h_pre), H_res = b_res + alpha_res tanh(Mat(h_res)),
 *   H_post = b_post + alpha_post tanh(h_post)   (no exp, no Sinkhorn, no sigmoid);
 * the read map is the same: x_in = sum_i H_pre[i] X[i, :].  work: [n*d + m] doubles. */
static void hc_pre_one_token(const double* Xt, const double* phi,
                             const double* b_pre, const double* b_post, const double* b_res,
                             double alpha_pre, double alpha_post, double alpha_res,
                             int n, int d, double eps, double* x_in_t, double* H_t, double* work)
{
    const int nd = n * d;
    const int m = n * n + 2 * n;
    double* xhat = work;          /* [nd] */
    double* h = xhat + nd;        /* [m]  */

    double ss = 0.0;
    for (int k = 0; k < nd; ++k) ss += Xt[k] * Xt[k];
    const double r = sqrt(ss / (double)nd + eps);
    for (int k = 0; k < nd; ++k) xhat[k] = Xt[k] / r;
    for (int j = 0; j < m; ++j) h[j] = 0.0;
    for (int k = 0; k < nd; ++k)
        for (int j = 0; j < m; ++j) h[j] += xhat[k] * phi[(long)k * m + j];

    for (int i = 0; i < n; ++i) H_t[i] = b_pre[i] + alpha_pre * tanh(h[i]);
    for (int k = 0; k < n * n; ++k) H_t[n + k] = b_res[k] + alpha_res * tanh(h[n + k]);
    for (int i = 0; i < n; ++i)
        H_t[n + n * n + i] = b_post[i] + alpha_post * tanh(h[n + n * n + i]);

    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += H_t[i] * Xt[i * d + c];
        x_in_t[c] = acc;
    }
}

void oracle_hc_pre(const double* X, const double* phi,
                   const double* b_pre, const double* b_post, const double* b_res,
                   double alpha_pre, double alpha_post, double alpha_res,
                   long T, int n, int d, double eps, double* x_in, double* H, int nthreads)
{
    const int nd = n * d;
    const int m = n * n + 2 * n;
    if (nthreads <= 0) nthreads = 1;
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* work = (double*)malloc(sizeof(double) * (size_t)(nd + m));
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
        for (long t = 0; t < T; ++t)
            hc_pre_one_token(X + t * (long)nd, phi, b_pre, b_post, b_res,
                             alpha_pre, alpha_post, alpha_res, n, d, eps,
                             x_in + t * (long)d, H + t * (long)m, work);
        free(work);
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

/* The normalised projection h = x_hat . phi of every token (the first two steps of the
 * pre stage, equations rmsnorm and the projection of the "DeepSeek-V4/mhc" page).
 * h [T, m]. */
void oracle_mhc_projection(const double* X, const double* phi, long T, int n, int d,
                           double eps, double* h, int nthreads)
{
    const int nd = n * d;
    const int m = n * n + 2 * n;
    if (nthreads <= 0) nthreads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (long t = 0; t < T; ++t) {
        const double* Xt = X + t * (long)nd;
        double* ht = h + t * (long)m;
        double ss = 0.0;
        for (int k = 0; k < nd; ++k) ss += Xt[k] * Xt[k];
        const double r = sqrt(ss / (double)nd + eps);
        for (int j = 0; j < m; ++j) ht[j] = 0.0;
        for (int k = 0; k < nd; ++k)
            for (int j = 0; j < m; ++j) ht[j] += (Xt[k] / r) * phi[(long)k * m + j];
    }
}

/* Reverse mode through one token of pre + post (the chain rule applied to the forward
 * steps above, last step first).  Besides dX and dF_out of the token it returns what the
 * token adds to the parameter gradients: dl [m], the gradient of the logits (ordered
 * [pre | res | post], also the token's term of db), dh [m] = alpha dl, the gradient of the
 * projection h, ga [3], the token's terms of dalpha (pre, post, res: the order of the
 * alpha arguments), and its RMS r, so that its term of dphi is (X_t / r) dh^T.
 * work: [nd (x_hat) + nd (dx_hat) + m (h) + n*n*(2*t_max+1) (iterates) + 2*n*n]. */
static void backward_one_token(const double* Xt, const double* Ft, const double* phi,
                               const double* b_pre, const double* b_post, const double* b_res,
                               double alpha_pre, double alpha_post, double alpha_res,
                               int n, int d, double eps, int t_max,
                               const double* dYt, const double* dxt,
                               double* dXt, double* dFt, double* dl, double* dh, double* ga,
                               double* r_out, double* work)
{
    const int nd = n * d, nn = n * n, m = nn + 2 * n;
    double* xhat = work;
    double* dxhat = xhat + nd;
    double* h = dxhat + nd;
    double* it = h + m;                   /* iterates M^(0..2 t_max), each n*n */
    double* gM = it + nn * (2 * t_max + 1);
    double* gA = gM + nn;

    /* ---- forward, keeping what the reverse sweep needs */
    double ss = 0.0;
    for (int k = 0; k < nd; ++k) ss += Xt[k] * Xt[k];
    const double r = sqrt(ss / (double)nd + eps);
    *r_out = r;
    for (int k = 0; k < nd; ++k) xhat[k] = Xt[k] / r;
    for (int j = 0; j < m; ++j) h[j] = 0.0;
    for (int k = 0; k < nd; ++k)
        for (int j = 0; j < m; ++j) h[j] += xhat[k] * phi[(long)k * m + j];
    double Hpre[8], Hpost[8];
    for (int i = 0; i < n; ++i) Hpre[i] = sigmoid(alpha_pre * h[i] + b_pre[i]);
    for (int i = 0; i < n; ++i) Hpost[i] = 2.0 * sigmoid(alpha_post * h[n + nn + i] + b_post[i]);
    for (int q = 0; q < nn; ++q) it[q] = exp(alpha_res * h[n + q] + b_res[q]);
    for (int s = 0; s < t_max; ++s) {
        const double* A = it + (2 * s) * nn;
        double* B = it + (2 * s + 1) * nn;      /* after the column step */
        double* C = it + (2 * s + 2) * nn;      /* after the row step    */
        for (int j = 0; j < n; ++j) {
            double cs = 0.0;
            for (int i = 0; i < n; ++i) cs += A[i * n + j];
            for (int i = 0; i < n; ++i) B[i * n + j] = A[i * n + j] / cs;
        }
        for (int i = 0; i < n; ++i) {
            double rs = 0.0;
            for (int j = 0; j < n; ++j) rs += B[i * n + j];
            for (int j = 0; j < n; ++j) C[i * n + j] = B[i * n + j] / rs;
        }
    }
    const double* Hres = it + (2 * t_max) * nn;

    /* ---- post: X' = H_res X + H_post^T F */
    for (int k = 0; k < nd; ++k) dXt[k] = 0.0;
    for (int q = 0; q < nn; ++q) gM[q] = 0.0;
    double dHpost[8], dHpre[8];
    for (int i = 0; i < n; ++i) {
        dHpost[i] = 0.0;
        for (int c = 0; c < d; ++c) dHpost[i] += dYt[i * d + c] * Ft[c];
        for (int j = 0; j < n; ++j)
            for (int c = 0; c < d; ++c) gM[i * n + j] += dYt[i * d + c] * Xt[j * d + c];
    }
    for (int j = 0; j < n; ++j)
        for (int c = 0; c < d; ++c)
            for (int i = 0; i < n; ++i) dXt[j * d + c] += Hres[i * n + j] * dYt[i * d + c];
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += Hpost[i] * dYt[i * d + c];
        dFt[c] = acc;
    }
    /* ---- read map: x_in = H_pre X */
    for (int i = 0; i < n; ++i) {
        dHpre[i] = 0.0;
        for (int c = 0; c < d; ++c) dHpre[i] += dxt[c] * Xt[i * d + c];
        for (int c = 0; c < d; ++c) dXt[i * d + c] += Hpre[i] * dxt[c];
    }
    /* ---- gates: sigmoid' = s (1 - s); H_post = 2 s */
    for (int i = 0; i < n; ++i) dl[i] = dHpre[i] * Hpre[i] * (1.0 - Hpre[i]);
    for (int i = 0; i < n; ++i) {
        const double s = 0.5 * Hpost[i];
        dl[n + nn + i] = dHpost[i] * 2.0 * s * (1.0 - s);
    }
    /* ---- Sinkhorn, last half-step first.  B = A / (row or column sum):
     *      dA = (dB - <dB, B> over that row or column) / sum */
    for (int s = t_max - 1; s >= 0; --s) {
        const double* A = it + (2 * s) * nn;
        const double* B = it + (2 * s + 1) * nn;
        const double* C = it + (2 * s + 2) * nn;
        for (int i = 0; i < n; ++i) {            /* row step: C = B / rowsum(B) */
            double rs = 0.0, dot = 0.0;
            for (int j = 0; j < n; ++j) { rs += B[i * n + j]; dot += gM[i * n + j] * C[i * n + j]; }
            for (int j = 0; j < n; ++j) gA[i * n + j] = (gM[i * n + j] - dot) / rs;
        }
        for (int j = 0; j < n; ++j) {            /* column step: B = A / colsum(A) */
            double cs = 0.0, dot = 0.0;
            for (int i = 0; i < n; ++i) { cs += A[i * n + j]; dot += gA[i * n + j] * B[i * n + j]; }
            for (int i = 0; i < n; ++i) gM[i * n + j] = (gA[i * n + j] - dot) / cs;
        }
    }
    for (int q = 0; q < nn; ++q) dl[n + q] = gM[q] * it[q];      /* M0 = exp(l_res) */
    /* ---- logits l = alpha h + b: db gets dl, dalpha gets <dl, h> per group */
    ga[0] = ga[1] = ga[2] = 0.0;
    for (int i = 0; i < n; ++i) { ga[0] += dl[i] * h[i]; dh[i] = alpha_pre * dl[i]; }
    for (int q = 0; q < nn; ++q) { ga[2] += dl[n + q] * h[n + q]; dh[n + q] = alpha_res * dl[n + q]; }
    for (int i = 0; i < n; ++i) {
        ga[1] += dl[n + nn + i] * h[n + nn + i];
        dh[n + nn + i] = alpha_post * dl[n + nn + i];
    }
    /* ---- projection h = x_hat phi (dphi gets x_hat dh^T, summed by the caller) */
    for (int k = 0; k < nd; ++k) {
        double acc = 0.0;
        for (int j = 0; j < m; ++j) acc += phi[(long)k * m + j] * dh[j];
        dxhat[k] = acc;
    }
    /* ---- RMSNorm x_hat = v / r, r = sqrt(sum v^2 / nd + eps) */
    double dot = 0.0;
    for (int k = 0; k < nd; ++k) dot += dxhat[k] * Xt[k];
    for (int k = 0; k < nd; ++k)
        dXt[k] += dxhat[k] / r - Xt[k] * dot / ((double)nd * r * r * r);
}

void oracle_mhc_backward(const double* X, const double* F_out, const double* phi,
                         const double* b_pre, const double* b_post, const double* b_res,
                         double alpha_pre, double alpha_post, double alpha_res,
                         long T, int n, int d, double eps, int t_max,
                         const double* dX_out, const double* dx_in,
                         double* dX, double* dF_out, double* dphi,
                         double* db_pre, double* db_post, double* db_res, double* dalpha,
                         int nthreads)
{
    const int nd = n * d, nn = n * n, m = nn + 2 * n;
    if (nthreads <= 0) nthreads = 1;
    const size_t wlen = (size_t)(2 * nd + m + nn * (2 * t_max + 1) + 2 * nn);
    /* per-token terms of the parameter gradients */
    double* dl = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * m);
    double* dh = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * m);
    double* ga = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * 3);
    double* rt = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* work = (double*)malloc(sizeof(double) * wlen);
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
        for (long t = 0; t < T; ++t)
            backward_one_token(X + t * (long)nd, F_out + t * (long)d, phi, b_pre, b_post, b_res,
                               alpha_pre, alpha_post, alpha_res, n, d, eps, t_max,
                               dX_out + t * (long)nd, dx_in + t * (long)d,
                               dX + t * (long)nd, dF_out + t * (long)d, dl + t * (long)m,
                               dh + t * (long)m, ga + 3 * t, rt + t, work);
        free(work);
    }
    /* The parameter gradients are sums over the tokens, each taken in token order:
     * dphi[k][j] = sum_t (X_t[k] / r_t) dh_t[j], db = sum_t dl_t, dalpha = sum_t ga_t.
     * Threads split the entries of dphi, never a sum, so the thread count does not
     * change any result. */
#ifdef _OPENMP
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (long k0 = 0; k0 < nd; k0 += 8) {            /* 8 entries of a row of X per pass */
        const int kb = (nd - k0) < 8 ? (int)(nd - k0) : 8;
        double acc[8][8 * 8 + 16];
        for (int u = 0; u < kb; ++u)
            for (int j = 0; j < m; ++j) acc[u][j] = 0.0;
        for (long t = 0; t < T; ++t)
            for (int u = 0; u < kb; ++u) {
                const double xh = X[t * (long)nd + k0 + u] / rt[t];
                for (int j = 0; j < m; ++j) acc[u][j] += xh * dh[t * (long)m + j];
            }
        for (int u = 0; u < kb; ++u)
            for (int j = 0; j < m; ++j) dphi[(k0 + u) * (long)m + j] = acc[u][j];
    }
    for (int j = 0; j < m; ++j) {
        double s = 0.0;
        for (long t = 0; t < T; ++t) s += dl[t * (long)m + j];
        if (j < n) db_pre[j] = s;
        else if (j < n + nn) db_res[j - n] = s;
        else db_post[j - n - nn] = s;
    }
    for (int a = 0; a < 3; ++a) {
        double s = 0.0;
        for (long t = 0; t < T; ++t) s += ga[3 * t + a];
        dalpha[a] = s;
    }
    free(dl);
    free(dh);
    free(ga);
    free(rt);
}

/* Amax Gain Magnitude of the composite residual maps ("DeepSeek-V4/mhc" page, the
 * stability paragraph: the largest absolute row sum -- forward -- and column sum --
 * backward -- of prod_{i=1..l} H_res of layer l+1-i; the slavadubrov.com article's numpy
 * demo forms the same product as C_l = H_res,l C_{l-1}).  Hs [L, T, m] holds each layer's
 * coefficient rows as written by the pre stage (H_res at offset n); gain [L, T, 2]
 * receives (forward, backward) of C_l for every prefix l = 1..L. */
void oracle_amax_gain(const double* Hs, int L, long T, int n, double* gain)
{
    const int m = n * n + 2 * n;
    double C[64], P[64];
    for (long t = 0; t < T; ++t) {
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) C[i * n + j] = (i == j) ? 1.0 : 0.0;
        for (int l = 0; l < L; ++l) {
            const double* A = Hs + ((long)l * T + t) * m + n;
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < n; ++j) {
                    double s = 0.0;
                    for (int q = 0; q < n; ++q) s += A[i * n + q] * C[q * n + j];
                    P[i * n + j] = s;
                }
            memcpy(C, P, sizeof(double) * (size_t)(n * n));
            double fwd = 0.0, bwd = 0.0;
            for (int i = 0; i < n; ++i) {
                double r = 0.0, c = 0.0;
                for (int j = 0; j < n; ++j) { r += fabs(C[i * n + j]); c += fabs(C[j * n + i]); }
                if (r > fwd) fwd = r;
                if (c > bwd) bwd = c;
            }
            gain[((long)l * T + t) * 2 + 0] = fwd;
            gain[((long)l * T + t) * 2 + 1] = bwd;
        }
    }
}
