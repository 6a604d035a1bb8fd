// launch.cuh -- internal launcher interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mhc {

enum DType { F32 = 0, BF16 = 1 };

struct PreArgs {
    const void* X;
    const float* phi;
    const float* b_pre;
    const float* b_post;
    const float* b_res;
    float a_pre, a_post, a_res;
    int64_t T;
    int n, d;
    float eps;
    int t_max;
    DType dt;
    void* x_in;
    float* H;
    float* h_out = nullptr;      // optional [T, m]: the normalised projection, for the backward
    bool hc = false;             // HC maps (bias + alpha tanh) instead of mHC's
    cudaStream_t stream;
};

struct PostArgs {
    const void* X;
    const void* F;
    const float* H;
    int64_t T;
    int n, d;
    DType dt;
    void* Y;
    cudaStream_t stream;
};

// Per-device launch limits, queried once per device and cached.
struct DeviceInfo {
    int device;
    int sm_count;
    int max_smem_optin;
    int cc_major, cc_minor;
};
cudaError_t device_info(DeviceInfo* out);

cudaError_t launch_pre_generic(const PreArgs& a);

// Tensor-core path (16-CTA clusters): shape test (host only) and launch.
bool pre_tc_shape_ok(int64_t T, int n, int d, DType dt);
// Whether the current device can run it for (n, d) (sm_100, phi slice fits shared memory,
// a resident 16-CTA cluster).
bool pre_tc_device_ok(int n, int d);
cudaError_t launch_pre_tc(const PreArgs& a);
// Status word of the tensor-core kernel's bounded waits (0 = fine); optionally cleared.
cudaError_t pre_tc_status(unsigned* out, bool clear);
// Failure-path test hook: launches after this call stop loading after `stop_tile` tiles
// per cluster (< 0: never) and give up a wait after `wait_ns`.
void pre_tc_set_stop(int stop_tile, unsigned long long wait_ns);

// Two-pass tensor-core path (8-CTA clusters, phi packed into the x_in buffer): shapes whose phi
// slice does not fit one 16-CTA cluster (n = 5..8, or n <= 4 with a large d).  The shape test
// includes the x_in buffer being large enough to hold the packed phi and the partials.
bool pre_wide_shape_ok(int64_t T, int n, int d, DType dt);
bool pre_wide_device_ok(int n);
cudaError_t launch_pre_wide(const PreArgs& a);
cudaError_t pre_wide_status(unsigned* out, bool clear);

cudaError_t launch_post(const PostArgs& a);

// Launch with programmatic stream serialisation: the kernel may start while the previous
// kernel on the stream finishes; it must execute pdl_wait() before it reads or writes any
// memory the previous work touches (without the attribute pdl_wait is a no-op).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
// wait for the previous kernel on the stream to complete and its memory to be visible
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// let the next kernel on the stream (launched with launch_pdl) start its own prologue
__device__ __forceinline__ void pdl_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Reverse mode of pre + post (backward.cu).
struct BwdArgs {
    const void* X;
    const void* F;
    const float* phi;
    const float* b_res;
    float a_pre, a_post, a_res;
    const float* H;              // forward coefficients [T, m]
    const float* h;              // saved normalised projection [T, m]
    int64_t T;
    int n, d;
    float eps;
    int t_max;
    DType dt;
    const void* dX_out;
    const void* dx_in;
    void* dX;
    void* dF_out;
    float* dphi;
    float* db_pre;
    float* db_post;
    float* db_res;
    float* dalpha;
    void* workspace;
    cudaStream_t stream;
};

// Workspace regions, in floats from the (256-byte aligned) workspace base.  The tensor-core
// dX / dphi step (tc) reads per-token records instead of G and beta.
struct BwdLayout {
    int64_t off_R, off_dl, off_G, off_beta, off_rec, off_part, off_colsum, floats;
    int groups;                  // token groups of the dX / dphi kernel
    int64_t tokens_per_group;
    bool tc;
};
BwdLayout backward_layout(int64_t T, int n, int d, bool tc);
// workspace the backward needs whichever dX / dphi kernel it takes, in floats
int64_t backward_workspace_floats(int64_t T, int n, int d);

// Tensor-core dX / dphi step (backward_tc.cu): bf16, n <= 4, d a multiple of 64.  It reads, per
// tile of BWD_REC_TILE tokens (token t in tile t / 64, row r = t % 64), a block of records written
// by the token kernel: bytes [0, 8192) hold row r's [G_hi | G_lo] (bf16, 32 each, zero past m)
// and bytes [8192, 16384) row r's per-stream fp32 coefficients {H_pre[i], H_res[0..3][i], -beta,
// 0, 0} for i < 4 (zero past n); each 128-byte row stores its 16-byte chunk j at position
// j ^ (r % 8), the 128-byte swizzle the MMA reads.  Rows past T are zero.
constexpr int BWD_REC_BYTES = 256;
constexpr int BWD_REC_TILE = 64;
constexpr int BWD_TC_SMS = 148;   // groups are sized for this many SMs (results do not depend on the device)
bool bwd_tc_shape_ok(int64_t T, int n, int d, DType dt);
bool bwd_tc_device_ok(int n);
int bwd_tc_groups(int64_t T, int d, int sm_count);
int64_t bwd_tc_tokens_per_group(int64_t T, int groups);
cudaError_t launch_bwd_tc(const BwdArgs& a, const void* rec, float* part, int groups, int64_t tpg);
cudaError_t bwd_tc_status(unsigned* out, bool clear);
// Failure-path test hook: launches after this call stop loading after `stop_stage` stages
// per CTA (< 0: never) and give up a wait after `wait_ns`.
void bwd_tc_set_stop(int stop_stage, unsigned long long wait_ns);

// Amax Gain Magnitude of composite residual maps (diagnostics.cu).
cudaError_t launch_amax_gain(const float* Hs, int L, int64_t T, int n, float* gain, cudaStream_t s);
cudaError_t launch_backward(const BwdArgs& a);

}  // namespace mhc
