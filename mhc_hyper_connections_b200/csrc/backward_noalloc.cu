// backward_noalloc.cu -- mhc_backward for callers that may not allocate device memory.
//
// mhc_backward needs a caller-owned workspace.  Some callers have no way to get one: code
// that only receives device pointers from a host framework which owns every device
// allocation through its own pool (a plugin, a C host with a fixed memory budget), or code
// for which a cudaMalloc -- which can synchronise the device -- is not allowed at the call
// site.  mhc_backward_noalloc serves them: it runs the same kernels with the workspace in a
// fixed array that is part of the library's device image, so the call itself allocates
// nothing.
#include <cuda.h>

#include <mutex>

#include "launch.cuh"
#include "mhc.h"

namespace mhc {

mhc_status report_cuda_error(cudaError_t e, const char* where);   // mhc_api.cu

namespace {

// The workspace of every mhc_backward_noalloc call on a device.  MHC_NOALLOC_SCRATCH_BYTES
// bytes; every device on which the library's code is loaded holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MHC_NOALLOC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Identifier of the context current on this thread (0 if none or if the driver cannot say).
// Resolved through the runtime, so the library does not link the driver library.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        cudaGetLastError();
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_noalloc_scratch on the current device.  In host code the array's name
// stands for a host-side shadow, not the device memory, so the address is looked up with the
// device current and cached per device and CUDA context: a device reset (or any new context
// on the device) gets a fresh lookup instead of a stale address.  When the driver cannot
// name the context, the address is looked up on every call.
cudaError_t scratch_address(void** out) {
    constexpr int kMaxDev = 64;
    static std::mutex mu;
    static void* addr[kMaxDev];
    static unsigned long long ctx_of[kMaxDev] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    const unsigned long long ctx = current_context_id();
    if (ctx == 0 || ctx != ctx_of[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // creates the context if needed
        if (e != cudaSuccess) return e;
        addr[dev] = p;
        ctx_of[dev] = current_context_id();
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
    // mhc_backward does every check in its own order; a size beyond the array fails its
    // workspace check (MHC_ERR_WORKSPACE) after the pointer, shape and alignment checks.
    void* scratch = nullptr;
    if (T > 0) {
        cudaError_t e = mhc::scratch_address(&scratch);
        if (e != cudaSuccess) return mhc::report_cuda_error(e, "mhc_backward_noalloc (scratch address)");
    }
    return mhc_backward(X, F_out, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, H, h,
                        T, n, d, eps, t_max, dt, dX_out, dx_in, dX, dF_out, dphi, db_pre, db_post,
                        db_res, dalpha, scratch, (size_t)MHC_NOALLOC_SCRATCH_BYTES, stream);
}
