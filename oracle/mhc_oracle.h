/*
 * mhc_oracle.h -- fp64 CPU oracle for the mHC layer (pre and post stages).
 *
 * TEST INFRASTRUCTURE ONLY.  This oracle exists to check the CUDA path.  Only
 * the test suite, the package smoke check and the benchmark's CPU-baseline /
 * reference leg may load it.  The product path never calls it and has no CPU
 * fallback.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (plain definitions, fp64 throughout):
 *   Dynamic parameterisation, "DeepSeek-V4/mhc" knowledge page, section
 *   "动态参数化怎么实现", equations rmsnorm and a/b/c-tilde:
 *     x_hat = RMSNorm(vec(X))                      (vec = row-stacked, index i*d+c)
 *     h     = x_hat . phi                          (phi columns: [pre | res | post])
 *     l_pre = alpha_pre  * h[0:n]        + b_pre
 *     l_res = alpha_res  * Mat(h[n:n+n^2]) + b_res (Mat = row-major n x n)
 *     l_post= alpha_post * h[n+n^2:m]    + b_post
 *   Gates, same page, equation "gate"; also the slavadubrov.com mHC article,
 *   section "Details van de parameterisatie":
 *     H_pre = sigmoid(l_pre), H_post = 2 * sigmoid(l_post)
 *   Sinkhorn-Knopp, same page, equations sinkhorn-init / sinkhorn; the
 *   slavadubrov.com article, section "Sinkhorn-Knopp-projectie":
 *     M = exp(l_res); repeat t_max times: divide every column by its sum, then
 *     every row by its sum; H_res = M.
 *   Layer update, slavadubrov.com article, "Kernmechanismen" (Eq. 3 of the
 *   paper), and the knowledge page's HC update equation:
 *     x_in = H_pre X           (raw X, not x_hat)
 *     X'   = H_res X + H_post^T F_out
 *
 * m = n*n + 2n.  The coefficient block H of one token is [H_pre | H_res | H_post].
 * All arrays are contiguous row-major host arrays of double.
 */
#ifndef MHC_ORACLE_H
#define MHC_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

/* exp(logits) then t_max rounds of (column normalisation, row normalisation).
 * logits, out: [n*n] row-major.  out may not alias logits. */
void oracle_sinkhorn(const double* logits, int n, int t_max, double* out);

/* Pre stage over T tokens.
 * X [T, n, d]; phi [n*d, m]; b_pre [n]; b_post [n]; b_res [n*n].
 * Outputs: x_in [T, d]; H [T, m] = [H_pre | H_res row-major | H_post].
 * nthreads <= 0 means one thread. */
void oracle_mhc_pre(const double* X, const double* phi,
                    const double* b_pre, const double* b_post, const double* b_res,
                    double alpha_pre, double alpha_post, double alpha_res,
                    long T, int n, int d, double eps, int t_max,
                    double* x_in, double* H, int nthreads);

/* HC pre stage (the unconstrained maps mHC is compared with) over T tokens: the same
 * RMSNorm and projection h, then H_pre = b_pre + alpha_pre tanh(h_pre),
 * H_res = b_res + alpha_res tanh(Mat(h_res)), H_post = b_post + alpha_post tanh(h_post),
 * and x_in = H_pre X.  Same layouts as oracle_mhc_pre; the post stage is oracle_mhc_post. */
void oracle_hc_pre(const double* X, const double* phi,
                   const double* b_pre, const double* b_post, const double* b_res,
                   double alpha_pre, double alpha_post, double alpha_res,
                   long T, int n, int d, double eps, double* x_in, double* H, int nthreads);

/* Post stage over T tokens: X_out[t,i,c] = sum_j H_res[i][j] X[t,j,c] + H_post[i] F_out[t,c].
 * X [T, n, d]; F_out [T, d]; H [T, m] as written by oracle_mhc_pre; X_out [T, n, d]. */
void oracle_mhc_post(const double* X, const double* F_out, const double* H,
                     long T, int n, int d, double* X_out, int nthreads);

/* The normalised projection h = RMSNorm(vec X_t) . phi of every token: h [T, m]. */
void oracle_mhc_projection(const double* X, const double* phi, long T, int n, int d,
                           double eps, double* h, int nthreads);

/* Reverse mode of pre + post for the loss L = <dX_out, X'> + <dx_in, x_in>, i.e. the
 * gradients of every input given the upstream gradients dX_out [T, n, d] (of X') and
 * dx_in [T, d] (of x_in).  The chain rule applied to the forward's steps in reverse
 * order; the Sinkhorn rounds are recomputed from the logits and their iterates kept in
 * scratch.  Outputs: dX [T, n, d] (through the projection, RMSNorm, the read map and the
 * merge), dF_out [T, d], dphi [n*d, m], db_pre [n], db_post [n], db_res [n*n] and
 * dalpha [3] = (pre, post, res) -- the order of the alpha arguments -- the parameter
 * gradients summed over all T tokens, each sum taken in token order (threads split the
 * tokens' own terms and the entries of dphi, never a sum). */
void oracle_mhc_backward(const double* X, const double* F_out, const double* phi,
                         const double* b_pre, const double* b_post, const double* b_res,
                         double alpha_pre, double alpha_post, double alpha_res,
                         long T, int n, int d, double eps, int t_max,
                         const double* dX_out, const double* dx_in,
                         double* dX, double* dF_out, double* dphi,
                         double* db_pre, double* db_post, double* db_res, double* dalpha,
                         int nthreads);

/* Amax Gain Magnitude of the composite residual maps C_l = H_res,l ... H_res,1 for every
 * prefix l of a stack of L layers: Hs [L, T, m] (each layer's coefficient rows), gain
 * [L, T, 2] = (largest absolute row sum, largest absolute column sum) of C_l.  n <= 8. */
void oracle_amax_gain(const double* Hs, int L, long T, int n, double* gain);

/* Number of OpenMP threads a parallel region with the given request uses. */
int oracle_threads_used(int nthreads);

#ifdef __cplusplus
}
#endif
#endif
