// common.cuh -- small device helpers shared by the mHC kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mhc {

// ---- element conversion ---------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// bf16 pair packed in a 32-bit word: element 0 in the low half.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---- 16-byte global accesses ------------------------------------------------------------
// Streaming read of data used once: read-only path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// A bf16 pair packed in a 32-bit word as an fp32 pair (element 0 first).
__device__ __forceinline__ float2 bf16x2_to_f32x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Unpack / pack a 16-byte vector of VEC elements to / from fp32.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int VEC = 4;
    __device__ __forceinline__ static void unpack(uint4 v, float* f) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int VEC = 8;
    __device__ __forceinline__ static void unpack(uint4 v, float* f) {
        f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
        f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                          pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
    }
};

// ---- the per-token maps (fp32) -------------------------------------------------------------
// sigmoid for H_pre, 2*sigmoid for H_post ("DeepSeek-V4/mhc", equation gate).
__device__ __forceinline__ float sigmoid_f32(float z) { return 1.0f / (1.0f + expf(-z)); }

// Sinkhorn-Knopp on an N x N matrix that already holds exp(logits) ("DeepSeek-V4/mhc",
// equation sinkhorn): t_max rounds of T_c (columns to sum 1) then T_r (rows to sum 1).
template <int N>
__device__ __forceinline__ void sinkhorn_rounds(float (&M)[N][N], int t_max) {
    for (int it = 0; it < t_max; ++it) {
#pragma unroll
        for (int j = 0; j < N; ++j) {
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < N; ++i) s += M[i][j];
            const float inv = 1.0f / s;
#pragma unroll
            for (int i = 0; i < N; ++i) M[i][j] *= inv;
        }
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < N; ++j) s += M[i][j];
            const float inv = 1.0f / s;
#pragma unroll
            for (int j = 0; j < N; ++j) M[i][j] *= inv;
        }
    }
}

// From the projection h (length m, NOT yet divided by r) to the coefficient block
// [H_pre | H_res | H_post] of one token ("DeepSeek-V4/mhc", equations a/b/c-tilde, gate,
// sinkhorn-init, sinkhorn).  The 1/r of RMSNorm is applied here, after the projection
// (the re-ordered RMSNorm of the infrastructure section).
template <int N>
__device__ __forceinline__ void token_maps(const float* h, float inv_r, const float* b_pre,
                                           const float* b_post, const float* b_res,
                                           float a_pre, float a_post, float a_res,
                                           int t_max, float* out) {
    constexpr int MM = N * N + 2 * N;
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = sigmoid_f32(a_pre * (h[i] * inv_r) + b_pre[i]);
    float Mx[N][N];
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int j = 0; j < N; ++j)
            Mx[i][j] = expf(a_res * (h[N + i * N + j] * inv_r) + b_res[i * N + j]);
    sinkhorn_rounds<N>(Mx, t_max);
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int j = 0; j < N; ++j) out[N + i * N + j] = Mx[i][j];
#pragma unroll
    for (int i = 0; i < N; ++i)
        out[N + N * N + i] = 2.0f * sigmoid_f32(a_post * (h[N + N * N + i] * inv_r) + b_post[i]);
    (void)MM;
}

// The HC maps mHC is compared with (slavadubrov.com article, "Kernmechanismen": a static
// bias plus an input-dependent term through tanh): every coefficient is
// b + alpha * tanh(h / r), with no sigmoid, exp or Sinkhorn.  Same layout as token_maps.
template <int N>
__device__ __forceinline__ void token_maps_hc(const float* h, float inv_r, const float* b_pre,
                                              const float* b_post, const float* b_res,
                                              float a_pre, float a_post, float a_res, float* out) {
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = b_pre[i] + a_pre * tanhf(h[i] * inv_r);
#pragma unroll
    for (int k = 0; k < N * N; ++k) out[N + k] = b_res[k] + a_res * tanhf(h[N + k] * inv_r);
#pragma unroll
    for (int i = 0; i < N; ++i)
        out[N + N * N + i] = b_post[i] + a_post * tanhf(h[N + N * N + i] * inv_r);
}

}  // namespace mhc
