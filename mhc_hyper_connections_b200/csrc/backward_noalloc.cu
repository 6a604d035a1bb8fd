// backward_noalloc.cu -- mhc_backward for callers that may not allocate device memory.
//
// mhc_backward needs a caller-owned workspace.  Some callers have no way to get one: code
// that only receives device pointers from a host framework which owns every device
// allocation through its own pool (a plugin, a C host with a fixed memory budget), or code
// for which a cudaMalloc -- which can synchronise the device -- is not allowed at the call
// site.  mhc_backward_noalloc serves them: it runs the same kernels with the workspace in a
// fixed array that is part of the library's device image, so the call itself allocates
// nothing.
#include <mutex>

#include "launch.cuh"
#include "mhc.h"

namespace mhc {

mhc_status report_cuda_error(cudaError_t e, const char* where);   // mhc_api.cu

namespace {

// The workspace of every mhc_backward_noalloc call on a device.  MHC_NOALLOC_SCRATCH_BYTES
// bytes; every device on which the library's code is loaded holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MHC_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code the array's name
// stands for a host-side shadow, not the device memory, so the address is looked up once per
// device, with that device current, and cached.
cudaError_t scratch_address(void** out) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static void* addr[kMaxDev];
    static bool have[kMaxDev] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!have[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
        have[dev] = true;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace mhc

extern "C" mhc_status mhc_backward_noalloc(
    const void* X, const void* F_out, const float* phi, const float* b_pre, const float* b_post,
    const float* b_res, float alpha_pre, float alpha_post, float alpha_res, const float* H,
    const float* h, int64_t T, int n, int d, float eps, int t_max, mhc_dtype dt,
    const void* dX_out, const void* dx_in, void* dX, void* dF_out, float* dphi, float* db_pre,
    float* db_post, float* db_res, float* dalpha, mhc_stream_t stream) {
    void* scratch = nullptr;
    if (T > 0) {
        const size_t need = mhc_backward_workspace_bytes(T, n, d);
        // need == 0: a shape mhc_backward rejects; let it return the status
        if (need > (size_t)MHC_NOALLOC_SCRATCH_BYTES) return MHC_ERR_WORKSPACE;
        if (need > 0) {
            cudaError_t e = mhc::scratch_address(&scratch);
            if (e != cudaSuccess) return mhc::report_cuda_error(e, "mhc_backward_noalloc (scratch address)");
        }
    }
    return mhc_backward(X, F_out, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, H, h,
                        T, n, d, eps, t_max, dt, dX_out, dx_in, dX, dF_out, dphi, db_pre, db_post,
                        db_res, dalpha, scratch, (size_t)MHC_NOALLOC_SCRATCH_BYTES, stream);
}
