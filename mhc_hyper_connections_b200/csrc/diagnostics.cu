// diagnostics.cu -- the Amax Gain Magnitude of composite residual maps.
//
// "DeepSeek-V4/mhc" page, stability paragraph: the gain of the composite mapping
// prod_{i=1..l} H_res of layer l+1-i is its largest absolute row sum (forward signal) and
// its largest absolute column sum (backward gradient); the slavadubrov.com article's numpy
// demo forms the product the same way, C_l = H_res,l C_{l-1}.  Given the coefficient rows
// H of L consecutive layers (as mhc_pre writes them, stacked [L, T, m]), one thread per
// token carries C_l in registers through the layers and writes both gains of every prefix;
// each layer's H_res is loaded a few layers before it is used.
#include "common.cuh"
#include "launch.cuh"

namespace mhc {
namespace {

constexpr int AMAX_THREADS = 64;      // small blocks spread the tokens over every SM

// H_res of layer l for token t, loaded PD layers ahead of its use (the loads do not depend on the
// running product, so their latency overlaps the layers in between)
template <int N>
__device__ __forceinline__ void load_res(const float* __restrict__ Hs, int64_t T, int64_t t, int l, int L,
                                         float (&a)[N][N]) {
    constexpr int M = N * N + 2 * N;
    if (l < L) {
        const float* A = Hs + ((int64_t)l * T + t) * M + N;
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int j = 0; j < N; ++j) a[i][j] = __ldg(A + i * N + j);
    }
}

template <int N>
__global__ void __launch_bounds__(AMAX_THREADS)
amax_gain_kernel(const float* __restrict__ Hs, int L, int64_t T, float* __restrict__ gain) {
    constexpr int PD = N <= 2 ? 4 : (N <= 4 ? 3 : 1);     // lookahead, within the register budget
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T; t += stride) {
        float C[N][N];
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int j = 0; j < N; ++j) C[i][j] = i == j ? 1.f : 0.f;
        float ring[PD][N][N];
#pragma unroll
        for (int k = 0; k < PD; ++k) load_res<N>(Hs, T, t, k, L, ring[k]);
        for (int l = 0; l < L; ++l) {
            float a[N][N];
#pragma unroll
            for (int i = 0; i < N; ++i)
#pragma unroll
                for (int j = 0; j < N; ++j) a[i][j] = ring[0][i][j];
#pragma unroll
            for (int k = 0; k + 1 < PD; ++k)
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int j = 0; j < N; ++j) ring[k][i][j] = ring[k + 1][i][j];
            load_res<N>(Hs, T, t, l + PD, L, ring[PD - 1]);
            float P[N][N];
#pragma unroll
            for (int i = 0; i < N; ++i)
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    float s = 0.f;
#pragma unroll
                    for (int q = 0; q < N; ++q) s = fmaf(a[i][q], C[q][j], s);
                    P[i][j] = s;
                }
            float fwd = 0.f, bwd = 0.f;
#pragma unroll
            for (int i = 0; i < N; ++i) {
                float r = 0.f, c = 0.f;
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    C[i][j] = P[i][j];
                    r += fabsf(P[i][j]);
                    c += fabsf(P[j][i]);
                }
                fwd = fmaxf(fwd, r);
                bwd = fmaxf(bwd, c);
            }
            gain[((int64_t)l * T + t) * 2 + 0] = fwd;
            gain[((int64_t)l * T + t) * 2 + 1] = bwd;
        }
    }
}

template <int N>
cudaError_t launch_n(const float* Hs, int L, int64_t T, float* gain, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    int64_t blocks = (T + AMAX_THREADS - 1) / AMAX_THREADS;
    if (blocks > (int64_t)di.sm_count * 32) blocks = (int64_t)di.sm_count * 32;
    amax_gain_kernel<N><<<(unsigned)blocks, AMAX_THREADS, 0, s>>>(Hs, L, T, gain);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_amax_gain(const float* Hs, int L, int64_t T, int n, float* gain, cudaStream_t s) {
    switch (n) {
        case 1: return launch_n<1>(Hs, L, T, gain, s);
        case 2: return launch_n<2>(Hs, L, T, gain, s);
        case 3: return launch_n<3>(Hs, L, T, gain, s);
        case 4: return launch_n<4>(Hs, L, T, gain, s);
        case 5: return launch_n<5>(Hs, L, T, gain, s);
        case 6: return launch_n<6>(Hs, L, T, gain, s);
        case 7: return launch_n<7>(Hs, L, T, gain, s);
        case 8: return launch_n<8>(Hs, L, T, gain, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace mhc
