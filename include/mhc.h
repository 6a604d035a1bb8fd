/*
 * mhc.h -- C ABI of the B200 (sm_100a) mHC layer: the pre and post stages, their
 * backward, and the Amax gain diagnostic.
 *
 * mHC (Manifold-Constrained Hyper-Connections) keeps n residual streams per token,
 * X_t in R^{n x d}, and wraps every sub-layer F in two per-token stages:
 *
 *   pre   x_hat = RMSNorm(vec X_t)   h = x_hat . phi   (logits, gates, Sinkhorn)
 *         x_in  = H_pre X_t                      -> fed to the sub-layer F
 *   post  X'_t  = H_res X_t + H_post^T F_out_t    -> the next layer's residual
 *
 * Sources ("page" = the web page of that title):
 *   - "DeepSeek-V4/mhc" knowledge page, section "动态参数化怎么实现": equations
 *     rmsnorm, a-tilde, b-tilde, c-tilde (logits), gate (sigmoid / 2 sigmoid),
 *     sinkhorn-init and sinkhorn (t_max = 20); its mixed-precision table (phi GEMM
 *     at TF32 or better, X in bf16, RMSNorm and Sinkhorn in fp32); its I/O-cost
 *     table (the n^2 + 2n coefficients per token handed from pre to post).
 *   - "DeepSeek mHC: Manifold-Constrained Hyper-Connections" (slavadubrov.com),
 *     section "Kernmechanismen", Eq. 3: x_{l+1} = H_res x_l + H_post^T F(H_pre x_l);
 *     section "Details van de parameterisatie": H_pre in (0,1), H_post in (0,2).
 *
 * Conventions shared by every entry point
 *   - All data pointers are DEVICE pointers, except the activations of
 *     mhc_forward_host, which live in host memory.  The caller allocates and owns every
 *     buffer; the library allocates no device memory.  Between calls it keeps a
 *     per-device cache of kernel launch limits, the two copy streams of
 *     mhc_forward_host and, in its device image, the status word of the bounded waits
 *     (mhc_device_status) and the fixed scratch array of mhc_backward_noalloc.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Arguments are validated on the host before any launch; a rejected
 *     call launches nothing and returns a non-zero mhc_status.  MHC_ERR_CUDA means
 *     a launch failed; mhc_last_error() then describes it (per host thread).
 *   - Layouts are contiguous row-major:
 *       X, X_out   [T, n, d]   stream i of token t at X + (t*n + i)*d
 *       F_out, x_in[T, d]
 *       phi        [n*d, m]    fp32, row k = i*d + c (the row-stacked flatten of X_t),
 *                              columns [pre (n) | res (n*n, row-major) | post (n)]
 *       H          [T, m]      fp32, m = n*n + 2n, per token [H_pre | H_res | H_post],
 *                              H_res row-major: H_res[i][j] weights input stream j
 *                              into output stream i.
 *       b_pre [n], b_post [n], b_res [n*n] (row-major), all fp32.
 *   - `dt` is the storage type of X, F_out, x_in and X_out; phi, biases and H are
 *     always fp32.  Arithmetic is fp32 (the projection accumulates in fp32 with phi
 *     carried at 16 significant bits or more).
 *   - Limits: 1 <= n <= 8 (a library limit, not the method's), d >= 1, T >= 0,
 *     0 <= t_max <= 1000.  T == 0 returns MHC_OK and launches nothing.
 *   - Alignment: every array must be aligned to its element size (else
 *     MHC_ERR_ALIGN).  16-byte-aligned arrays with d a multiple of 16/sizeof(elem)
 *     take the vectorised kernels; others take a scalar kernel with the same results
 *     up to fp32 rounding order.
 *   - Aliasing: outputs may not overlap any input or each other (MHC_ERR_ALIAS).
 *   - NaN and Inf propagate; nothing on the hot path checks values.
 */
#ifndef MHC_H
#define MHC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                        /* = cudaStream_t without the CUDA headers */
typedef struct CUstream_st* mhc_stream_t;

typedef enum {
    MHC_OK = 0,
    MHC_ERR_NULL = 1,          /* a required pointer is NULL (with T > 0)            */
    MHC_ERR_SHAPE = 2,         /* n, d, T or t_max out of range, or size overflow    */
    MHC_ERR_ALIGN = 3,         /* a pointer is not aligned to its element size       */
    MHC_ERR_DTYPE = 4,         /* dt is not an mhc_dtype value                       */
    MHC_ERR_UNSUPPORTED = 5,   /* the requested kernel path cannot run this problem  */
    MHC_ERR_CUDA = 6,          /* a CUDA call or launch failed                       */
    MHC_ERR_ALIAS = 7,         /* an output overlaps an input or another output      */
    MHC_ERR_WORKSPACE = 8      /* workspace smaller than its *_workspace_bytes query  */
} mhc_status;

typedef enum { MHC_F32 = 0, MHC_BF16 = 1 } mhc_dtype;

/* Kernel paths of the pre stage (mhc_pre picks MHC_PRE_AUTO). */
typedef enum {
    MHC_PRE_AUTO = 0,          /* the fastest path that supports the problem          */
    MHC_PRE_GENERIC = 1,       /* CUDA-core kernel: any n <= 8, any d, f32 or bf16    */
    MHC_PRE_CLUSTER_TC = 2,    /* thread-block-cluster tensor-core kernel, X read     */
                               /* once (bf16, n <= 4, d % 64 == 0, n*d >= 1024, phi   */
                               /* slice fits shared memory: d <= 5632 at n = 4)       */
    MHC_PRE_TWO_PASS_TC = 3    /* tensor-core projection, then a streaming read map   */
                               /* (X read twice; bf16, n <= 8, d % 64 == 0,           */
                               /* n*d >= 512, and x_in large enough to hold phi       */
                               /* packed for the MMA plus the partial projections --  */
                               /* it is used as scratch before x_in is written)       */
} mhc_pre_path;

/*
 * mhc_pre -- the pre stage for T tokens.
 * Defined by the "DeepSeek-V4/mhc" page equations rmsnorm, a/b/c-tilde, gate,
 * sinkhorn-init and sinkhorn, and the read map H_pre x_l of the slavadubrov.com Eq. 3:
 *   r      = sqrt(mean_k v_k^2 + eps)              v = vec(X_t), k = i*d + c
 *   h      = (v / r) . phi                          [m]
 *   H_pre  = sigmoid(alpha_pre * h[0:n] + b_pre)
 *   H_res  = SK_{t_max}(exp(alpha_res * Mat(h[n:n+n^2]) + b_res))
 *            (each round: divide every column by its sum, then every row by its sum)
 *   H_post = 2 sigmoid(alpha_post * h[n+n^2:m] + b_post)
 *   x_in   = sum_i H_pre[i] X_t[i, :]               (raw X, not x_hat)
 * Inputs : X [T,n,d] (dt), phi [n*d, m], b_pre [n], b_post [n], b_res [n*n],
 *          alpha_*, eps (the page uses 1e-20), t_max (the page uses 20).
 * Outputs: x_in [T,d] (dt), H [T,m] (fp32) = [H_pre | H_res | H_post] per token.
 * Errors : see "Conventions"; MHC_ERR_CUDA if a launch fails.
 */
mhc_status mhc_pre(const void* X, const float* phi, const float* b_pre, const float* b_post,
                   const float* b_res, float alpha_pre, float alpha_post, float alpha_res,
                   int64_t T, int n, int d, float eps, int t_max, mhc_dtype dt,
                   void* x_in, float* H, mhc_stream_t stream);

/*
 * mhc_pre_with_path -- mhc_pre on an explicitly chosen kernel path (same arguments and
 * results).  Returns MHC_ERR_UNSUPPORTED, launching nothing, if `path` cannot run the
 * problem on the current device.
 */
mhc_status mhc_pre_with_path(const void* X, const float* phi, const float* b_pre,
                             const float* b_post, const float* b_res, float alpha_pre,
                             float alpha_post, float alpha_res, int64_t T, int n, int d,
                             float eps, int t_max, mhc_dtype dt, void* x_in, float* H,
                             mhc_stream_t stream, mhc_pre_path path);

/*
 * mhc_pre_hc -- the pre stage with the HC maps that mHC is compared with: the unconstrained
 * hyper-connections of the slavadubrov.com article, section "Kernmechanismen" (each map a
 * static bias plus an input-dependent term through tanh, entries of either sign; its
 * "Details van de parameterisatie" names tanh as what mHC replaces by the sigmoid).  The
 * input-dependent term is the same normalised projection h that mhc_pre computes:
 *   H_pre  = b_pre  + alpha_pre  * tanh(h[0:n])
 *   H_res  = b_res  + alpha_res  * tanh(Mat(h[n:n+n^2]))      (no exp, no Sinkhorn)
 *   H_post = b_post + alpha_post * tanh(h[n+n^2:m])
 *   x_in   = sum_i H_pre[i] X_t[i, :]
 * Same arguments, layouts, kernel paths and errors as mhc_pre_with_path, without t_max.
 * mhc_post applies the result unchanged; mhc_amax_gain measures how its composite
 * residual maps grow with depth, the comparison the pages draw.
 */
mhc_status mhc_pre_hc(const void* X, const float* phi, const float* b_pre, const float* b_post,
                      const float* b_res, float alpha_pre, float alpha_post, float alpha_res,
                      int64_t T, int n, int d, float eps, mhc_dtype dt, void* x_in, float* H,
                      mhc_stream_t stream, mhc_pre_path path);

/*
 * mhc_pre_path_for -- the path MHC_PRE_AUTO would take for this problem on the current
 * device (host-side query; launches nothing): MHC_PRE_CLUSTER_TC where it runs, else
 * MHC_PRE_TWO_PASS_TC where it runs, else MHC_PRE_GENERIC.  The tensor-core paths also
 * need X, x_in and phi 16-byte aligned; MHC_PRE_AUTO takes MHC_PRE_GENERIC when they are not.
 */
mhc_pre_path mhc_pre_path_for(int64_t T, int n, int d, mhc_dtype dt);

/*
 * mhc_pre_path_ok -- 1 if `path` can run a pre stage of this shape and storage type on the
 * current device (given 16-byte-aligned X, x_in and phi for the tensor-core paths), else 0.
 * MHC_PRE_AUTO and MHC_PRE_GENERIC run every valid shape.  Host-side, launches nothing.
 */
int mhc_pre_path_ok(int64_t T, int n, int d, mhc_dtype dt, mhc_pre_path path);

/*
 * mhc_post -- the post/res merge for T tokens (slavadubrov.com Eq. 3, first and second
 * term; the "Post-Res fused kernel" row of the knowledge page's kernel table, which
 * reads X and F_out once):
 *   X_out[t, i, :] = sum_j H_res[i][j] X[t, j, :] + H_post[i] F_out[t, :]
 * Inputs : X [T,n,d] (dt), F_out [T,d] (dt), H [T,m] fp32 as written by mhc_pre.
 * Output : X_out [T,n,d] (dt); may not alias X, F_out or H.
 */
mhc_status mhc_post(const void* X, const void* F_out, const float* H, int64_t T, int n, int d,
                    mhc_dtype dt, void* X_out, mhc_stream_t stream);

/*
 * mhc_forward_host -- mhc_pre, then mhc_post, for T tokens whose activations live in HOST
 * memory (slavadubrov.com Eq. 3 with the sub-layer's output F_out given, as mhc_post takes
 * it).  This is the one entry point with host pointers:
 *   host   : X_h [T,n,d], F_out_h [T,d] (inputs); x_in_h [T,d], H_h [T,m], X_out_h [T,n,d]
 *            (outputs), same layouts and dtypes as the device entry points.  Page-locked
 *            (pinned) host memory lets the copies overlap; pageable memory gives the same
 *            results with the copies serialised by the driver.
 *   device : phi, b_pre, b_post, b_res (the parameters stay resident on the device), and
 *            `workspace`, 256-byte aligned, at least
 *            mhc_forward_host_workspace_bytes(chunk_tokens, n, d, dt) bytes.  It may not
 *            overlap the parameters.
 * The tokens go through in chunks of chunk_tokens (the last chunk may be shorter), rotating
 * through three device buffer sets in the workspace. The copies into the device of chunk c+1,
 * the two stages on chunk c and the copies back of chunk c-1 overlap. The copies use two
 * streams of the library's own, created on the first call on a device and kept for the
 * process. Everything is ordered after the work already queued on `stream`, and `stream`
 * resumes only once every output has landed in host memory. So a host read of the outputs
 * needs a synchronisation of `stream`, and the workspace may be reused by the next call on
 * the same stream.
 * Every output of a token depends on that token alone, so the outputs are those of mhc_pre
 * and mhc_post called on each chunk. That is bit for bit the whole-batch result wherever the
 * chunk takes the same kernel path (mhc_pre_path_for).
 * Errors: the argument checks of mhc_pre, plus MHC_ERR_SHAPE for chunk_tokens < 1 (or a
 * chunk too large to address), MHC_ERR_WORKSPACE, and MHC_ERR_ALIAS for host outputs that
 * overlap a host input or each other, or a workspace that overlaps the parameters.  All of
 * them are checked before anything is queued.  A CUDA failure part-way (MHC_ERR_CUDA) leaves
 * the outputs incomplete, and copies already queued may still run: synchronise the device
 * before reusing the host buffers.  Calls on one device from several host threads are
 * serialised while they queue their work.
 */
size_t mhc_forward_host_workspace_bytes(int64_t chunk_tokens, int n, int d, mhc_dtype dt);

mhc_status mhc_forward_host(const void* X_h, const void* F_out_h, const float* phi,
                            const float* b_pre, const float* b_post, const float* b_res,
                            float alpha_pre, float alpha_post, float alpha_res, int64_t T, int n,
                            int d, float eps, int t_max, mhc_dtype dt, void* x_in_h, float* H_h,
                            void* X_out_h, int64_t chunk_tokens, void* workspace,
                            size_t workspace_bytes, mhc_stream_t stream);

/*
 * mhc_pre_train -- mhc_pre for training: the same computation and outputs, plus the
 * normalised projection of every token, which mhc_backward needs to re-form the logits:
 *   h[t, :] = (vec X_t / r_t) . phi                 [T, m] fp32, written in place
 * (the "DeepSeek-V4/mhc" page, equations rmsnorm and the projection; the logits of
 * equations a/b/c-tilde are alpha * h + b).  h may not overlap any other argument.
 */
mhc_status mhc_pre_train(const void* X, const float* phi, const float* b_pre, const float* b_post,
                         const float* b_res, float alpha_pre, float alpha_post, float alpha_res,
                         int64_t T, int n, int d, float eps, int t_max, mhc_dtype dt,
                         void* x_in, float* H, float* h, mhc_stream_t stream);

/*
 * mhc_backward_workspace_bytes -- device workspace mhc_backward needs for (T, n, d); 0 for
 * a shape it rejects.  Host-side, launches nothing.
 */
size_t mhc_backward_workspace_bytes(int64_t T, int n, int d);

/*
 * mhc_backward -- reverse mode of pre + post: the gradients of
 *   L = <dX_out, X'> + <dx_in, x_in>
 * with respect to X, F_out, phi, the biases and the three alphas, for the forward of
 * mhc_pre / mhc_post above (the chain rule through each step of the "DeepSeek-V4/mhc"
 * page's equations rmsnorm, a/b/c-tilde, gate, sinkhorn-init and sinkhorn, and the read
 * map and merge of the slavadubrov.com Eq. 3, last step first).  The Sinkhorn rounds are
 * recomputed from the pre-exp logits alpha_res * h_res + b_res; no iterate is stored.
 * Inputs : X [T,n,d], F_out [T,d] (dt); phi [n*d, m]; b_pre [n], b_post [n], b_res [n*n];
 *          alpha_*, eps, t_max as given to the forward; H [T,m] and h [T,m] as written by
 *          mhc_pre_train; dX_out [T,n,d] (gradient of X') and dx_in [T,d] (gradient of
 *          x_in), dt.
 * Outputs: dX [T,n,d] and dF_out [T,d] (dt); dphi [n*d, m], db_pre [n], db_post [n],
 *          db_res [n*n] and dalpha [3] = (pre, post, res), fp32, summed over all T tokens
 *          in a fixed order (repeated calls give bitwise equal results).  For T == 0 the
 *          parameter gradients are set to zero.
 * workspace: device memory of at least mhc_backward_workspace_bytes(T, n, d) bytes,
 *          256-byte aligned, owned by the caller, overwritten (else MHC_ERR_WORKSPACE).
 * Limits : n <= 4 (MHC_ERR_UNSUPPORTED above); X, F_out, dX_out, dx_in, dX and dF_out
 *          16-byte aligned with d * sizeof(element) a multiple of 16 (else MHC_ERR_ALIGN).
 *          No output may overlap an input or another output (MHC_ERR_ALIAS).
 * Kernels: bf16 with d a multiple of 64 runs the products phi G (for dX) and X^T G (dphi)
 *          on the tensor cores with G and phi split into bf16 hi + lo parts (16 significant
 *          bits each, fp32 accumulation); other shapes and fp32 run them on CUDA cores.
 */
mhc_status mhc_backward(const void* X, const void* F_out, const float* phi, const float* b_pre,
                        const float* b_post, const float* b_res, float alpha_pre, float alpha_post,
                        float alpha_res, const float* H, const float* h, int64_t T, int n, int d,
                        float eps, int t_max, mhc_dtype dt, const void* dX_out, const void* dx_in,
                        void* dX, void* dF_out, float* dphi, float* db_pre, float* db_post,
                        float* db_res, float* dalpha, void* workspace, size_t workspace_bytes,
                        mhc_stream_t stream);

/* Size of the fixed scratch array mhc_backward_noalloc works in: 32 MiB. */
#define MHC_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * mhc_backward_noalloc -- mhc_backward without a caller-provided workspace, for callers
 * that cannot allocate device memory: code that only receives device pointers from a host
 * framework which owns every allocation through its own memory pool, or a call site where
 * a cudaMalloc (which can synchronise the device) is not allowed.  The paper has no
 * counterpart to this; it is a library convenience.
 *
 * Same arguments, results and errors as mhc_backward, minus the workspace pair, and checked
 * in the same order.  The workspace is a fixed array of MHC_NOALLOC_SCRATCH_BYTES bytes
 * inside the library's device image: every device on which the library's code is loaded
 * holds it until the process exits, and the call itself allocates nothing (no cudaMalloc,
 * no cudaFree).
 *   - Sizes whose mhc_backward_workspace_bytes(T, n, d) exceeds MHC_NOALLOC_SCRATCH_BYTES
 *     fail mhc_backward's workspace check: MHC_ERR_WORKSPACE, after the pointer, shape and
 *     alignment checks, launching nothing (T = 16384, n = 4, d = 4096 needs 30.0 MB and
 *     fits).
 *   - The first call on a device (T > 0) looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it for the device's
 *     current CUDA context; a later context on the device (after cudaDeviceReset, say)
 *     gets a new lookup.  Make the first call on each device, and the first after a reset,
 *     before any stream capture on it.  If the lookup fails the call returns MHC_ERR_CUDA
 *     before any other check.
 *   - All calls on a device share the one array, which keeps whatever the last call left
 *     in it.  Nothing in it needs to start at zero (every kernel writes its part before
 *     reading it), but calls that overlap on the GPU -- on different streams, or from
 *     different host threads -- race on it: order them.
 */
mhc_status mhc_backward_noalloc(const void* X, const void* F_out, const float* phi,
                                const float* b_pre, const float* b_post, const float* b_res,
                                float alpha_pre, float alpha_post, float alpha_res,
                                const float* H, const float* h, int64_t T, int n, int d,
                                float eps, int t_max, mhc_dtype dt, const void* dX_out,
                                const void* dx_in, void* dX, void* dF_out, float* dphi,
                                float* db_pre, float* db_post, float* db_res, float* dalpha,
                                mhc_stream_t stream);

/*
 * mhc_amax_gain -- the Amax Gain Magnitude of the composite residual maps of L consecutive
 * layers ("DeepSeek-V4/mhc" page, stability paragraph; the slavadubrov.com article's numpy
 * demo): for every token and every prefix l = 1..L of the stack,
 *   C_l = H_res(layer l) . H_res(layer l-1) ... H_res(layer 1)
 *   gain[l-1, t, 0] = max_i sum_j |C_l[i][j]|   (forward: largest absolute row sum)
 *   gain[l-1, t, 1] = max_j sum_i |C_l[i][j]|   (backward: largest absolute column sum)
 * A diagnostic of depth-wise stability, not part of the layer's hot path.
 * Inputs : H_layers [L, T, m] fp32, the coefficient rows mhc_pre wrote for each layer,
 *          stacked (layer l at H_layers + l*T*m); 1 <= n <= 8, L >= 0, T >= 0.
 * Output : gain [L, T, 2] fp32, written in place; may not overlap H_layers.
 * L == 0 or T == 0 returns MHC_OK and launches nothing.
 */
mhc_status mhc_amax_gain(const float* H_layers, int L, int64_t T, int n, float* gain,
                         mhc_stream_t stream);

/*
 * mhc_device_status -- read and clear the device-side status words of the tensor-core
 * kernels.  Their waits between warps and between the CTAs of a cluster are bounded in
 * time (1 s each); a wait that expires makes the kernel stop early, leaving its outputs
 * incomplete, and sets a bit here naming the wait: bits 0-15 the cluster pre kernel, 16-23
 * the two-pass pre kernels, 24-31 the tensor-core dX / dphi step of mhc_backward.  *code = 0
 * means every wait of every launch since the last read completed.  Blocks until prior work on the legacy default
 * stream (and streams that synchronise with it) has finished.  No counterpart on the
 * pages: this is the library's failure report.
 */
mhc_status mhc_device_status(uint32_t* code);

/*
 * mhc_debug_pre_stop_after -- test hook for the failure path of the tensor-core pre kernel
 * (MHC_PRE_CLUSTER_TC).  After this call, its launches stop loading X after `tiles` token
 * tiles per cluster (tiles < 0: never, the default) and give up a wait after
 * `wait_limit_us` microseconds (default 1000000; accepted range 1000 .. 10000000, else
 * MHC_ERR_SHAPE).  Every cluster stops at the same tile boundary, so all the tiles before
 * it complete; the waits that depend on the tiles never loaded run into their limit, the
 * kernel sets bits in mhc_device_status, drains its own copies in flight (those drain
 * waits keep a limit of at least 1 s) and returns with x_in and H incomplete.  The setting
 * is process-wide and applies from the next launch.  No counterpart on the pages: a
 * library test facility for the bounded waits.
 */
mhc_status mhc_debug_pre_stop_after(int32_t tiles, uint32_t wait_limit_us);

/*
 * mhc_debug_backward_stop_after -- test hook for the failure path of mhc_backward's
 * tensor-core dX / dphi step (bf16, d a multiple of 64).  After this call its launches stop
 * loading after `stages` 64-token stages per CTA (stages < 0: never, the default) and give
 * up a wait after `wait_limit_us` microseconds (default 1000000; accepted range 1000 ..
 * 10000000, else MHC_ERR_SHAPE).  Every stage before the stop completes (its dX tile is
 * stored); the waits for the stage never loaded run into their limit, the step sets bits
 * 24-31 in mhc_device_status, lets its copies and MMAs in flight complete and returns with dX
 * and the parameter gradients incomplete.  Process-wide, from the next launch.  No
 * counterpart on the pages: a library test facility for the bounded waits.
 */
mhc_status mhc_debug_backward_stop_after(int32_t stages, uint32_t wait_limit_us);

/* Static English text for a status code (never NULL). */
const char* mhc_status_string(mhc_status status);

/* Text of the last MHC_ERR_CUDA raised on the calling host thread ("" if none). */
const char* mhc_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MHC_H */
