// post.cu -- the mHC post/res merge X'_i = sum_j H_res[i][j] X_j + H_post[i] F_out.
//
// slavadubrov.com mHC article, "Kernmechanismen" Eq. 3 (residual term and block update);
// the "Post-Res fused kernel" of the "DeepSeek-V4/mhc" kernel table (X and F_out read
// once: (n+1) d elements in, n d out per token).
//
// Pure streaming, HBM bound.  Vector kernel: one warp task = one token x 32 chunks of 16
// bytes (8 bf16 / 4 fp32 channels); every lane loads its chunk of the n streams and of
// F_out with 16-byte read-only loads, mixes in fp32 and stores n 16-byte chunks.  The
// token's n^2 + n coefficients are warp-uniform loads served from L1.  A persistent grid
// of (SMs x resident CTAs) strides over the tasks.
#include "common.cuh"
#include "launch.cuh"

namespace mhc {
namespace {

constexpr int THREADS = 256;

// HV: H is 16-byte aligned and its rows are a multiple of 16 bytes long.
template <int N, bool HV>
__device__ __forceinline__ void load_coeffs(const float* __restrict__ Ht, float (&hr)[N][N],
                                            float (&hp)[N]) {
    if constexpr (HV) {
        // rows of H are 16-byte aligned: the H_res/H_post part starts at float N
        float buf[N * N + N + (N % 4 ? 4 - N % 4 : 0) + 4];
        const int base = N & ~3;                       // 16-byte aligned start <= N
        constexpr int cnt = ((N + N * N + N) - (N & ~3) + 3) / 4;
#pragma unroll
        for (int q = 0; q < cnt; ++q) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(Ht + base) + q);
            buf[4 * q + 0] = v.x; buf[4 * q + 1] = v.y; buf[4 * q + 2] = v.z; buf[4 * q + 3] = v.w;
        }
        const int off = N - base;
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int j = 0; j < N; ++j) hr[i][j] = buf[off + i * N + j];
#pragma unroll
        for (int i = 0; i < N; ++i) hp[i] = buf[off + N * N + i];
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int j = 0; j < N; ++j) hr[i][j] = __ldg(Ht + N + i * N + j);
#pragma unroll
        for (int i = 0; i < N; ++i) hp[i] = __ldg(Ht + N + N * N + i);
    }
}

// Launched plainly, after the previous work on the stream has finished: with a programmatic
// dependent launch (griddepcontrol.wait at the top) the n = 8 instance compiled to 182 registers
// instead of 128 and streamed at 70 % of the copy bandwidth instead of 90 %.
template <int N, typename T, bool HV>
__global__ void __launch_bounds__(THREADS)
post_vec_kernel(const T* __restrict__ X, const T* __restrict__ F, const float* __restrict__ H,
                int64_t Tn, int d, T* __restrict__ Y)
{
    constexpr int M = N * N + 2 * N;
    constexpr int VEC = Vec16<T>::VEC;
    const int chunks = d / VEC;
    const int tasks_per_tok = (chunks + 31) >> 5;
    const int64_t ntasks = Tn * tasks_per_tok;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t task = (((int64_t)blockIdx.x * blockDim.x) + threadIdx.x) >> 5; task < ntasks;
         task += nwarps) {
        const int64_t t = task / tasks_per_tok;
        const int q = (int)(task - t * tasks_per_tok) * 32 + lane;
        float hr[N][N], hp[N];
        load_coeffs<N, HV>(H + t * M, hr, hp);
        if (q < chunks) {
            uint4 xv[N];
#pragma unroll
            for (int i = 0; i < N; ++i)
                xv[i] = ld_stream_v4(X + (t * N + i) * (int64_t)d + (int64_t)q * VEC);
            const uint4 fv = ld_stream_v4(F + t * (int64_t)d + (int64_t)q * VEC);
            float xf[N][VEC], ff[VEC];
#pragma unroll
            for (int i = 0; i < N; ++i) Vec16<T>::unpack(xv[i], xf[i]);
            Vec16<T>::unpack(fv, ff);
#pragma unroll
            for (int i = 0; i < N; ++i) {
                float o[VEC];
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    float a = hr[i][0] * xf[0][e];
#pragma unroll
                    for (int j = 1; j < N; ++j) a = fmaf(hr[i][j], xf[j][e], a);
                    o[e] = fmaf(hp[i], ff[e], a);
                }
                st_v4(Y + (t * N + i) * (int64_t)d + (int64_t)q * VEC, Vec16<T>::pack(o));
            }
        }
    }
}

// Any d / alignment: one thread per (token, channel), all n streams.
template <int N, typename T>
__global__ void __launch_bounds__(THREADS)
post_scalar_kernel(const T* __restrict__ X, const T* __restrict__ F, const float* __restrict__ H,
                   int64_t Tn, int d, T* __restrict__ Y)
{
    constexpr int M = N * N + 2 * N;
    const int64_t total = Tn * d;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
        const int64_t t = e / d;
        const int c = (int)(e - t * d);
        const float* Ht = H + t * M;
        float xf[N];
#pragma unroll
        for (int j = 0; j < N; ++j) xf[j] = to_f32(X[(t * N + j) * (int64_t)d + c]);
        const float f = to_f32(F[t * (int64_t)d + c]);
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float a = __ldg(Ht + N + i * N) * xf[0];
#pragma unroll
            for (int j = 1; j < N; ++j) a = fmaf(__ldg(Ht + N + i * N + j), xf[j], a);
            store_elem(&Y[(t * N + i) * (int64_t)d + c], fmaf(__ldg(Ht + N + N * N + i), f, a));
        }
    }
}

template <int N, typename T>
cudaError_t launch_n(const PostArgs& a) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    constexpr int VEC = Vec16<T>::VEC;
    const bool vec = (a.d % VEC == 0) && ((uintptr_t)a.X % 16 == 0) &&
                     ((uintptr_t)a.F % 16 == 0) && ((uintptr_t)a.Y % 16 == 0);
    constexpr int M = N * N + 2 * N;
    const bool hv = ((M * 4) % 16 == 0) && ((uintptr_t)a.H % 16 == 0);
    if (vec) {
        auto kern = hv ? post_vec_kernel<N, T, ((M * 4) % 16 == 0)> : post_vec_kernel<N, T, false>;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, 0);
        if (e != cudaSuccess) return e;
        const int64_t tasks = a.T * (((a.d / VEC) + 31) / 32);
        const int64_t want = (tasks * 32 + THREADS - 1) / THREADS;
        const int64_t cap = (int64_t)di.sm_count * (per_sm > 0 ? per_sm : 1);
        const unsigned blocks = (unsigned)(want < cap ? want : cap);
        kern<<<blocks, THREADS, 0, a.stream>>>(static_cast<const T*>(a.X), static_cast<const T*>(a.F), a.H,
                                                a.T, a.d, static_cast<T*>(a.Y));
    } else {
        const int64_t want = (a.T * a.d + THREADS - 1) / THREADS;
        const int64_t cap = (int64_t)di.sm_count * 8;
        const unsigned blocks = (unsigned)(want < cap ? want : cap);
        post_scalar_kernel<N, T><<<blocks, THREADS, 0, a.stream>>>(
            static_cast<const T*>(a.X), static_cast<const T*>(a.F), a.H, a.T, a.d, static_cast<T*>(a.Y));
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const PostArgs& a) {
    switch (a.n) {
        case 1: return launch_n<1, T>(a);
        case 2: return launch_n<2, T>(a);
        case 3: return launch_n<3, T>(a);
        case 4: return launch_n<4, T>(a);
        case 5: return launch_n<5, T>(a);
        case 6: return launch_n<6, T>(a);
        case 7: return launch_n<7, T>(a);
        case 8: return launch_n<8, T>(a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_post(const PostArgs& a) {
    return a.dt == BF16 ? launch_t<__nv_bfloat16>(a) : launch_t<float>(a);
}

}  // namespace mhc
