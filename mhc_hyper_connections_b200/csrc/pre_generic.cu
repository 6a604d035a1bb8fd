// pre_generic.cu -- CUDA-core kernel for the mHC pre stage: any n <= 8, any d, f32 or bf16.
//
// Per CTA a tile of TT tokens:
//   1. K loop (K = n*d): stage X[tile, k0:k0+KC] (as fp32) and phi[k0:k0+KC, :] in shared
//      memory; accumulate the projection h = v . phi (fp32; each thread a TM-token by
//      ceil(m/32)-column register tile) and the sum of squares of v.
//   2. One thread per token turns h into [H_pre | H_res | H_post] ("DeepSeek-V4/mhc",
//      equations rmsnorm, a/b/c-tilde, gate, sinkhorn; or the HC maps, bias + alpha tanh)
//      and writes H.
//   3. x_in = sum_i H_pre[i] X[t, i, :] (slavadubrov.com Eq. 3, read map on raw X).
// Exact fp32 arithmetic with fp32 phi: this is the path for fp32 storage and for shapes
// the tensor-core path does not take.
#include "common.cuh"
#include "launch.cuh"

namespace mhc {
namespace {

constexpr int TT = 32;        // tokens per CTA
constexpr int KC = 32;        // K chunk staged per step
constexpr int THREADS = 256;
constexpr int TM = 4;         // tokens of a thread's projection micro-tile
constexpr int JS = THREADS / (TT / TM);     // column groups: thread columns j = jg + JS * q

template <int N, typename T>
__global__ void __launch_bounds__(THREADS)
pre_generic_kernel(const T* __restrict__ X, const float* __restrict__ phi,
                   const float* __restrict__ b_pre, const float* __restrict__ b_post,
                   const float* __restrict__ b_res, float a_pre, float a_post, float a_res,
                   int64_t Tn, int d, float eps, int t_max, T* __restrict__ x_in,
                   float* __restrict__ H, float* __restrict__ h_out, int hc)
{
    constexpr int M = N * N + 2 * N;
    constexpr int TJ = (M + JS - 1) / JS;              // columns per thread
    constexpr int SPT = KC * TT / THREADS;             // X elements staged per thread
    __shared__ float xs[TT][KC + 1];
    __shared__ float ps[KC][JS * TJ];                  // columns past M hold zeros
    __shared__ float hs[TT][M];
    __shared__ float ss_s[TT];
    __shared__ float hpre_s[TT][N];

    const int K = N * d;
    const int64_t t0 = (int64_t)blockIdx.x * TT;
    const int tid = threadIdx.x;
    const int tg = tid / JS, jg = tid % JS;             // micro-tile: tokens tg*TM.., columns jg + JS*q

    float acc[TM][TJ];
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int q = 0; q < TJ; ++q) acc[a][q] = 0.f;
    float ssq = 0.f;                                  // partial sum of squares of token my_t
    const int my_t = tid / (THREADS / TT);            // THREADS / TT threads per token when staging
    const int my_k0 = (tid % (THREADS / TT)) * SPT;
    const int64_t my_tok = t0 + my_t;

    // chunk k0's X and phi values travel through registers: the next chunk's loads are in
    // flight while this chunk is multiplied
    constexpr int PPT = (KC * JS * TJ + THREADS - 1) / THREADS;   // phi values staged per thread
    float xr[SPT], pr[PPT];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int u = 0; u < SPT; ++u) {
            const int k = k0 + my_k0 + u;
            xr[u] = (my_tok < Tn && k < K) ? to_f32(X[my_tok * K + k]) : 0.f;
        }
#pragma unroll
        for (int r = 0; r < PPT; ++r) {
            const int e = tid + THREADS * r;
            const int kk = e / (JS * TJ), j = e - kk * (JS * TJ);
            const int k = k0 + kk;
            pr[r] = (e < KC * JS * TJ && k < K && j < M) ? phi[(int64_t)k * M + j] : 0.f;
        }
    };
    fetch(0);
    for (int k0 = 0; k0 < K; k0 += KC) {
#pragma unroll
        for (int u = 0; u < SPT; ++u) {
            xs[my_t][my_k0 + u] = xr[u];
            ssq = fmaf(xr[u], xr[u], ssq);
        }
#pragma unroll
        for (int r = 0; r < PPT; ++r) {
            const int e = tid + THREADS * r;
            if (e < KC * JS * TJ) ps[e / (JS * TJ)][e % (JS * TJ)] = pr[r];
        }
        __syncthreads();
        if (k0 + KC < K) fetch(k0 + KC);
#pragma unroll 4
        for (int kk = 0; kk < KC; ++kk) {
            float xv[TM], pv[TJ];
#pragma unroll
            for (int a = 0; a < TM; ++a) xv[a] = xs[tg * TM + a][kk];
#pragma unroll
            for (int q = 0; q < TJ; ++q) pv[q] = ps[kk][jg + JS * q];
#pragma unroll
            for (int a = 0; a < TM; ++a)
#pragma unroll
                for (int q = 0; q < TJ; ++q) acc[a][q] = fmaf(xv[a], pv[q], acc[a][q]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < TM; ++a)
#pragma unroll
        for (int q = 0; q < TJ; ++q) {
            const int j = jg + JS * q;
            if (j < M) hs[tg * TM + a][j] = acc[a][q];
        }
    // sum of squares: the THREADS / TT threads of a token are consecutive lanes
#pragma unroll
    for (int off = THREADS / TT / 2; off > 0; off >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
    if ((tid % (THREADS / TT)) == 0) ss_s[my_t] = ssq;
    __syncthreads();

    if (tid < TT && t0 + tid < Tn) {
        const int64_t tok = t0 + tid;
        const float r = sqrtf(ss_s[tid] / (float)K + eps);
        float out[M];
        const float inv_r = 1.0f / r;
        if (hc) token_maps_hc<N>(hs[tid], inv_r, b_pre, b_post, b_res, a_pre, a_post, a_res, out);
        else token_maps<N>(hs[tid], inv_r, b_pre, b_post, b_res, a_pre, a_post, a_res, t_max, out);
#pragma unroll
        for (int j = 0; j < M; ++j) H[tok * M + j] = out[j];
        if (h_out != nullptr) {        // the normalised projection, as the logits use it
#pragma unroll
            for (int j = 0; j < M; ++j) h_out[tok * M + j] = hs[tid][j] * inv_r;
        }
#pragma unroll
        for (int i = 0; i < N; ++i) hpre_s[tid][i] = out[i];
    }
    __syncthreads();

    for (int e = tid; e < TT * d; e += THREADS) {
        const int t = e / d, c = e - t * d;
        const int64_t tok = t0 + t;
        if (tok >= Tn) break;
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < N; ++i) a = fmaf(hpre_s[t][i], to_f32(X[tok * K + (int64_t)i * d + c]), a);
        store_elem(&x_in[tok * d + c], a);
    }
}

template <int N, typename T>
cudaError_t launch_n(const PreArgs& a) {
    const int64_t blocks = (a.T + TT - 1) / TT;
    if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
    pre_generic_kernel<N, T><<<(unsigned)blocks, THREADS, 0, a.stream>>>(
        static_cast<const T*>(a.X), a.phi, a.b_pre, a.b_post, a.b_res, a.a_pre, a.a_post,
        a.a_res, a.T, a.d, a.eps, a.t_max, static_cast<T*>(a.x_in), a.H, a.h_out, a.hc ? 1 : 0);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const PreArgs& a) {
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

cudaError_t launch_pre_generic(const PreArgs& a) {
    return a.dt == BF16 ? launch_t<__nv_bfloat16>(a) : launch_t<float>(a);
}

}  // namespace mhc
