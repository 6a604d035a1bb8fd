// mhc_api.cu -- the C ABI declared in include/mhc.h: host-side validation and dispatch.
//
// Every argument is checked on the host before anything is launched; a rejected call
// launches nothing.  The library allocates no device memory.
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "launch.cuh"
#include "mhc.h"

namespace mhc {

static thread_local char g_last_error[256] = "";

static mhc_status cuda_fail(cudaError_t e, const char* where) {
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(e),
             cudaGetErrorString(e));
    return MHC_ERR_CUDA;
}

// Records a CUDA error for mhc_last_error and returns MHC_ERR_CUDA (for other C-ABI files).
mhc_status report_cuda_error(cudaError_t e, const char* where) { return cuda_fail(e, where); }

cudaError_t device_info(DeviceInfo* out) {
    constexpr int kMaxDev = 64;
    static DeviceInfo cache[kMaxDev];
    static bool valid[kMaxDev] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!valid[dev]) {
        DeviceInfo di{};
        di.device = dev;
        if ((e = cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&di.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&di.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return e;
        cache[dev] = di;
        valid[dev] = true;
    }
    *out = cache[dev];
    return cudaSuccess;
}

}  // namespace mhc

using namespace mhc;

namespace {

size_t elem_size(mhc_dtype dt) { return dt == MHC_BF16 ? 2 : 4; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (na == 0 || nb == 0) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Common shape checks; also rejects sizes whose byte counts would overflow int64.
mhc_status check_shape(int64_t T, int n, int d, mhc_dtype dt) {
    if (dt != MHC_F32 && dt != MHC_BF16) return MHC_ERR_DTYPE;
    if (n < 1 || n > 8 || d < 1 || T < 0) return MHC_ERR_SHAPE;
    const int64_t row = (int64_t)n * d;                     // elements per token
    if (row > (int64_t)1 << 30) return MHC_ERR_SHAPE;       // phi rows and K fit in int
    if (T > (((int64_t)1 << 62) / (row * 8))) return MHC_ERR_SHAPE;
    return MHC_OK;
}

mhc_status validate_pre(const void* X, const float* phi, const float* b_pre, const float* b_post,
                        const float* b_res, int64_t T, int n, int d, int t_max, mhc_dtype dt,
                        const void* x_in, const float* H) {
    mhc_status st = check_shape(T, n, d, dt);
    if (st != MHC_OK) return st;
    if (t_max < 0 || t_max > 1000) return MHC_ERR_SHAPE;
    if (T == 0) return MHC_OK;
    if (!X || !phi || !b_pre || !b_post || !b_res || !x_in || !H) return MHC_ERR_NULL;
    const size_t es = elem_size(dt);
    if (!aligned(X, es) || !aligned(x_in, es) || !aligned(phi, 4) || !aligned(b_pre, 4) ||
        !aligned(b_post, 4) || !aligned(b_res, 4) || !aligned(H, 4))
        return MHC_ERR_ALIGN;
    const int m = n * n + 2 * n;
    const size_t nX = (size_t)T * n * d * es, nxin = (size_t)T * d * es, nH = (size_t)T * m * 4;
    const size_t nphi = (size_t)n * d * m * 4;
    const void* ins[5] = {X, phi, b_pre, b_post, b_res};
    const size_t nins[5] = {nX, nphi, (size_t)n * 4, (size_t)n * 4, (size_t)n * n * 4};
    for (int i = 0; i < 5; ++i)
        if (overlaps(x_in, nxin, ins[i], nins[i]) || overlaps(H, nH, ins[i], nins[i]))
            return MHC_ERR_ALIAS;
    if (overlaps(x_in, nxin, H, nH)) return MHC_ERR_ALIAS;
    return MHC_OK;
}

PreArgs make_pre(const void* X, const float* phi, const float* b_pre, const float* b_post,
                 const float* b_res, float a_pre, float a_post, float a_res, int64_t T, int n,
                 int d, float eps, int t_max, mhc_dtype dt, void* x_in, float* H,
                 mhc_stream_t stream) {
    PreArgs a;
    a.X = X; a.phi = phi; a.b_pre = b_pre; a.b_post = b_post; a.b_res = b_res;
    a.a_pre = a_pre; a.a_post = a_post; a.a_res = a_res;
    a.T = T; a.n = n; a.d = d; a.eps = eps; a.t_max = t_max;
    a.dt = dt == MHC_BF16 ? BF16 : F32;
    a.x_in = x_in; a.H = H;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    return a;
}

}  // namespace

extern "C" {

mhc_pre_path mhc_pre_path_for(int64_t T, int n, int d, mhc_dtype dt) {
    if (check_shape(T, n, d, dt) != MHC_OK) return MHC_PRE_GENERIC;
    const DType t = dt == MHC_BF16 ? BF16 : F32;
    if (pre_tc_shape_ok(T, n, d, t) && pre_tc_device_ok(n, d)) return MHC_PRE_CLUSTER_TC;
    if (pre_wide_shape_ok(T, n, d, t) && pre_wide_device_ok(n)) return MHC_PRE_TWO_PASS_TC;
    return MHC_PRE_GENERIC;
}

int mhc_pre_path_ok(int64_t T, int n, int d, mhc_dtype dt, mhc_pre_path path) {
    if (check_shape(T, n, d, dt) != MHC_OK) return 0;
    const DType t = dt == MHC_BF16 ? BF16 : F32;
    switch (path) {
        case MHC_PRE_AUTO:
        case MHC_PRE_GENERIC: return 1;
        case MHC_PRE_CLUSTER_TC: return pre_tc_shape_ok(T, n, d, t) && pre_tc_device_ok(n, d);
        case MHC_PRE_TWO_PASS_TC: return pre_wide_shape_ok(T, n, d, t) && pre_wide_device_ok(n);
    }
    return 0;
}

static mhc_status pre_impl(const void* X, const float* phi, const float* b_pre, const float* b_post,
                           const float* b_res, float alpha_pre, float alpha_post, float alpha_res,
                           int64_t T, int n, int d, float eps, int t_max, mhc_dtype dt, void* x_in,
                           float* H, float* h_out, mhc_stream_t stream, mhc_pre_path path,
                           bool hc = false) {
    mhc_status st = validate_pre(X, phi, b_pre, b_post, b_res, T, n, d, t_max, dt, x_in, H);
    if (st != MHC_OK) return st;
    if (path != MHC_PRE_AUTO && path != MHC_PRE_GENERIC && path != MHC_PRE_CLUSTER_TC &&
        path != MHC_PRE_TWO_PASS_TC)
        return MHC_ERR_UNSUPPORTED;
    if (T == 0) return MHC_OK;
    const bool tc_aligned = aligned(X, 16) && aligned(x_in, 16) && aligned(phi, 16);
    if (path == MHC_PRE_AUTO) {
        path = mhc_pre_path_for(T, n, d, dt);
        if (path != MHC_PRE_GENERIC && !tc_aligned) path = MHC_PRE_GENERIC;
    }
    PreArgs a = make_pre(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, T,
                         n, d, eps, t_max, dt, x_in, H, stream);
    a.h_out = h_out;
    a.hc = hc;
    cudaError_t e;
    if (path == MHC_PRE_CLUSTER_TC) {
        if (!pre_tc_shape_ok(T, n, d, a.dt) || !pre_tc_device_ok(n, d) || !tc_aligned)
            return MHC_ERR_UNSUPPORTED;
        e = launch_pre_tc(a);
        if (e != cudaSuccess) return cuda_fail(e, "mhc_pre (tensor-core kernel)");
    } else if (path == MHC_PRE_TWO_PASS_TC) {
        if (!pre_wide_shape_ok(T, n, d, a.dt) || !pre_wide_device_ok(n) || !tc_aligned)
            return MHC_ERR_UNSUPPORTED;
        e = launch_pre_wide(a);
        if (e != cudaSuccess) return cuda_fail(e, "mhc_pre (two-pass tensor-core kernels)");
    } else {
        e = launch_pre_generic(a);
        if (e != cudaSuccess) return cuda_fail(e, "mhc_pre (generic kernel)");
    }
    return MHC_OK;
}

mhc_status mhc_pre_with_path(const void* X, const float* phi, const float* b_pre,
                             const float* b_post, const float* b_res, float alpha_pre,
                             float alpha_post, float alpha_res, int64_t T, int n, int d,
                             float eps, int t_max, mhc_dtype dt, void* x_in, float* H,
                             mhc_stream_t stream, mhc_pre_path path) {
    return pre_impl(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, T, n, d, eps,
                    t_max, dt, x_in, H, nullptr, stream, path);
}

mhc_status mhc_pre_hc(const void* X, const float* phi, const float* b_pre, const float* b_post,
                      const float* b_res, float alpha_pre, float alpha_post, float alpha_res,
                      int64_t T, int n, int d, float eps, mhc_dtype dt, void* x_in, float* H,
                      mhc_stream_t stream, mhc_pre_path path) {
    return pre_impl(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, T, n, d, eps,
                    0, dt, x_in, H, nullptr, stream, path, true);
}

mhc_status mhc_pre_train(const void* X, const float* phi, const float* b_pre, const float* b_post,
                         const float* b_res, float alpha_pre, float alpha_post, float alpha_res,
                         int64_t T, int n, int d, float eps, int t_max, mhc_dtype dt, void* x_in,
                         float* H, float* h, mhc_stream_t stream) {
    mhc_status st = check_shape(T, n, d, dt);
    if (st != MHC_OK) return st;
    if (T > 0) {
        if (!h) return MHC_ERR_NULL;
        if (!aligned(h, 4)) return MHC_ERR_ALIGN;
        const int m = n * n + 2 * n;
        const size_t es = elem_size(dt), nh = (size_t)T * m * 4;
        const void* other[7] = {X, phi, b_pre, b_post, b_res, x_in, H};
        const size_t nother[7] = {(size_t)T * n * d * es, (size_t)n * d * m * 4, (size_t)n * 4,
                                  (size_t)n * 4, (size_t)n * n * 4, (size_t)T * d * es, nh};
        for (int i = 0; i < 7; ++i)
            if (overlaps(h, nh, other[i], nother[i])) return MHC_ERR_ALIAS;
    }
    return pre_impl(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, T, n, d, eps,
                    t_max, dt, x_in, H, h, stream, MHC_PRE_AUTO);
}

size_t mhc_backward_workspace_bytes(int64_t T, int n, int d) {
    if (check_shape(T, n, d, MHC_F32) != MHC_OK || n > 4) return 0;
    return (size_t)backward_workspace_floats(T, n, d) * 4;
}

mhc_status mhc_backward(const void* X, const void* F_out, const float* phi, const float* b_pre,
                        const float* b_post, const float* b_res, float alpha_pre, float alpha_post,
                        float alpha_res, const float* H, const float* h, int64_t T, int n, int d,
                        float eps, int t_max, mhc_dtype dt, const void* dX_out, const void* dx_in,
                        void* dX, void* dF_out, float* dphi, float* db_pre, float* db_post,
                        float* db_res, float* dalpha, void* workspace, size_t workspace_bytes,
                        mhc_stream_t stream) {
    mhc_status st = check_shape(T, n, d, dt);
    if (st != MHC_OK) return st;
    if (t_max < 0 || t_max > 1000) return MHC_ERR_SHAPE;
    if (n > 4) return MHC_ERR_UNSUPPORTED;
    if (!phi || !b_pre || !b_post || !b_res || !dphi || !db_pre || !db_post || !db_res || !dalpha)
        return MHC_ERR_NULL;
    const int m = n * n + 2 * n;
    const size_t es = elem_size(dt);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t nphi = (size_t)n * d * m * 4;
    if (T == 0) {   // no tokens: every parameter gradient is zero
        cudaError_t e = cudaMemsetAsync(dphi, 0, nphi, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(db_pre, 0, (size_t)n * 4, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(db_post, 0, (size_t)n * 4, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(db_res, 0, (size_t)n * n * 4, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dalpha, 0, 3 * 4, s);
        return e == cudaSuccess ? MHC_OK : cuda_fail(e, "mhc_backward");
    }
    if (!X || !F_out || !H || !h || !dX_out || !dx_in || !dX || !dF_out || !workspace) return MHC_ERR_NULL;
    const void* vec[6] = {X, F_out, dX_out, dx_in, dX, dF_out};
    for (int i = 0; i < 6; ++i)
        if (!aligned(vec[i], 16)) return MHC_ERR_ALIGN;
    if ((size_t)d * es % 16 != 0) return MHC_ERR_ALIGN;
    const float* f4[9] = {phi, b_pre, b_post, b_res, H, h, dphi, db_pre, db_post};
    for (int i = 0; i < 9; ++i)
        if (!aligned(f4[i], 4)) return MHC_ERR_ALIGN;
    if (!aligned(db_res, 4) || !aligned(dalpha, 4) || !aligned(workspace, 256)) return MHC_ERR_ALIGN;
    const size_t need = mhc_backward_workspace_bytes(T, n, d);
    if (workspace_bytes < need) return MHC_ERR_WORKSPACE;
    const size_t nX = (size_t)T * n * d * es, nD = (size_t)T * d * es, nH = (size_t)T * m * 4;
    const void* ins[10] = {X, F_out, phi, b_pre, b_post, b_res, H, h, dX_out, dx_in};
    const size_t nins[10] = {nX, nD, nphi, (size_t)n * 4, (size_t)n * 4, (size_t)n * n * 4, nH, nH, nX, nD};
    void* outs[8] = {dX, dF_out, dphi, db_pre, db_post, db_res, dalpha, workspace};
    const size_t nouts[8] = {nX, nD, nphi, (size_t)n * 4, (size_t)n * 4, (size_t)n * n * 4, 12, need};
    for (int o = 0; o < 8; ++o) {
        for (int i = 0; i < 10; ++i)
            if (overlaps(outs[o], nouts[o], ins[i], nins[i])) return MHC_ERR_ALIAS;
        for (int p = o + 1; p < 8; ++p)
            if (overlaps(outs[o], nouts[o], outs[p], nouts[p])) return MHC_ERR_ALIAS;
    }
    BwdArgs a;
    a.X = X; a.F = F_out; a.phi = phi; a.b_res = b_res;
    a.a_pre = alpha_pre; a.a_post = alpha_post; a.a_res = alpha_res;
    a.H = H; a.h = h; a.T = T; a.n = n; a.d = d; a.eps = eps; a.t_max = t_max;
    a.dt = dt == MHC_BF16 ? BF16 : F32;
    a.dX_out = dX_out; a.dx_in = dx_in; a.dX = dX; a.dF_out = dF_out; a.dphi = dphi;
    a.db_pre = db_pre; a.db_post = db_post; a.db_res = db_res; a.dalpha = dalpha;
    a.workspace = workspace;
    a.stream = s;
    cudaError_t e = launch_backward(a);
    if (e != cudaSuccess) return cuda_fail(e, "mhc_backward");
    return MHC_OK;
}

mhc_status mhc_pre(const void* X, const float* phi, const float* b_pre, const float* b_post,
                   const float* b_res, float alpha_pre, float alpha_post, float alpha_res,
                   int64_t T, int n, int d, float eps, int t_max, mhc_dtype dt, void* x_in,
                   float* H, mhc_stream_t stream) {
    return mhc_pre_with_path(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, T, n,
                             d, eps, t_max, dt, x_in, H, stream, MHC_PRE_AUTO);
}

mhc_status mhc_post(const void* X, const void* F_out, const float* H, int64_t T, int n, int d,
                    mhc_dtype dt, void* X_out, mhc_stream_t stream) {
    mhc_status st = check_shape(T, n, d, dt);
    if (st != MHC_OK) return st;
    if (T == 0) return MHC_OK;
    if (!X || !F_out || !H || !X_out) return MHC_ERR_NULL;
    const size_t es = elem_size(dt);
    if (!aligned(X, es) || !aligned(F_out, es) || !aligned(X_out, es) || !aligned(H, 4))
        return MHC_ERR_ALIGN;
    const int m = n * n + 2 * n;
    const size_t nX = (size_t)T * n * d * es;
    if (overlaps(X_out, nX, X, nX) || overlaps(X_out, nX, F_out, (size_t)T * d * es) ||
        overlaps(X_out, nX, H, (size_t)T * m * 4))
        return MHC_ERR_ALIAS;
    PostArgs a;
    a.X = X; a.F = F_out; a.H = H; a.T = T; a.n = n; a.d = d;
    a.dt = dt == MHC_BF16 ? BF16 : F32;
    a.Y = X_out;
    a.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_post(a);
    if (e != cudaSuccess) return cuda_fail(e, "mhc_post");
    return MHC_OK;
}

mhc_status mhc_amax_gain(const float* H_layers, int L, int64_t T, int n, float* gain,
                         mhc_stream_t stream) {
    if (n < 1 || n > 8 || L < 0 || T < 0) return MHC_ERR_SHAPE;
    const int m = n * n + 2 * n;
    if (L > 0 && T > (((int64_t)1 << 58) / ((int64_t)L * m))) return MHC_ERR_SHAPE;
    if (L == 0 || T == 0) return MHC_OK;
    if (!H_layers || !gain) return MHC_ERR_NULL;
    if (!aligned(H_layers, 4) || !aligned(gain, 4)) return MHC_ERR_ALIGN;
    if (overlaps(gain, (size_t)L * T * 8, H_layers, (size_t)L * T * m * 4)) return MHC_ERR_ALIAS;
    cudaError_t e = launch_amax_gain(H_layers, L, T, n, gain, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "mhc_amax_gain");
    return MHC_OK;
}

const char* mhc_status_string(mhc_status s) {
    switch (s) {
        case MHC_OK: return "ok";
        case MHC_ERR_NULL: return "a required pointer is NULL";
        case MHC_ERR_SHAPE: return "n, d, T or t_max out of range";
        case MHC_ERR_ALIGN: return "a pointer is not aligned to its element size";
        case MHC_ERR_DTYPE: return "unknown dtype";
        case MHC_ERR_UNSUPPORTED: return "the requested kernel path cannot run this problem";
        case MHC_ERR_CUDA: return "a CUDA call or launch failed (see mhc_last_error)";
        case MHC_ERR_ALIAS: return "an output overlaps an input or another output";
        case MHC_ERR_WORKSPACE: return "the workspace is smaller than its *_workspace_bytes query";
    }
    return "unknown status";
}

const char* mhc_last_error(void) { return g_last_error; }

mhc_status mhc_debug_pre_stop_after(int32_t tiles, uint32_t wait_limit_us) {
    if (wait_limit_us < 1000u || wait_limit_us > 10000000u) return MHC_ERR_SHAPE;
    pre_tc_set_stop(tiles < 0 ? -1 : (int)tiles, (unsigned long long)wait_limit_us * 1000ull);
    return MHC_OK;
}

mhc_status mhc_debug_backward_stop_after(int32_t stages, uint32_t wait_limit_us) {
    if (wait_limit_us < 1000u || wait_limit_us > 10000000u) return MHC_ERR_SHAPE;
    bwd_tc_set_stop(stages < 0 ? -1 : (int)stages, (unsigned long long)wait_limit_us * 1000ull);
    return MHC_OK;
}

mhc_status mhc_device_status(uint32_t* code) {
    if (!code) return MHC_ERR_NULL;
    unsigned v = 0, w = 0, b = 0;
    cudaError_t e = pre_tc_status(&v, true);
    if (e == cudaSuccess) e = pre_wide_status(&w, true);
    if (e == cudaSuccess) e = bwd_tc_status(&b, true);
    if (e != cudaSuccess) return cuda_fail(e, "mhc_device_status");
    *code = v | (w << 16) | (b << 24);
    return MHC_OK;
}

}  // extern "C"
