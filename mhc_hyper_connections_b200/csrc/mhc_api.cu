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
    if (pre_cluster_tc_shape_ok(T, n, d, t) && pre_cluster_tc_device_ok(n, d)) return MHC_PRE_CLUSTER_TC;
    return MHC_PRE_GENERIC;
}

mhc_status mhc_pre_with_path(const void* X, const float* phi, const float* b_pre,
                             const float* b_post, const float* b_res, float alpha_pre,
                             float alpha_post, float alpha_res, int64_t T, int n, int d,
                             float eps, int t_max, mhc_dtype dt, void* x_in, float* H,
                             mhc_stream_t stream, mhc_pre_path path) {
    mhc_status st = validate_pre(X, phi, b_pre, b_post, b_res, T, n, d, t_max, dt, x_in, H);
    if (st != MHC_OK) return st;
    if (path != MHC_PRE_AUTO && path != MHC_PRE_GENERIC && path != MHC_PRE_CLUSTER_TC)
        return MHC_ERR_UNSUPPORTED;
    if (T == 0) return MHC_OK;
    if (path == MHC_PRE_AUTO) path = mhc_pre_path_for(T, n, d, dt);
    const PreArgs a = make_pre(X, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, T,
                               n, d, eps, t_max, dt, x_in, H, stream);
    cudaError_t e;
    if (path == MHC_PRE_CLUSTER_TC) {
        if (!pre_cluster_tc_shape_ok(T, n, d, a.dt) || !pre_cluster_tc_device_ok(n, d))
            return MHC_ERR_UNSUPPORTED;
        if (!aligned(X, 16) || !aligned(x_in, 16) || !aligned(phi, 16)) return MHC_ERR_UNSUPPORTED;
        e = launch_pre_cluster_tc(a);
        if (e != cudaSuccess) return cuda_fail(e, "mhc_pre (cluster tensor-core kernel)");
    } else {
        e = launch_pre_generic(a);
        if (e != cudaSuccess) return cuda_fail(e, "mhc_pre (generic kernel)");
    }
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
    }
    return "unknown status";
}

const char* mhc_last_error(void) { return g_last_error; }

mhc_status mhc_device_status(uint32_t* code) {
    if (!code) return MHC_ERR_NULL;
    unsigned v = 0;
    cudaError_t e = pre_cluster_tc_status(&v, true);
    if (e != cudaSuccess) return cuda_fail(e, "mhc_device_status");
    *code = v;
    return MHC_OK;
}

}  // extern "C"
