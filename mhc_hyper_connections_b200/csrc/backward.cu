// backward.cu -- reverse mode of the mHC layer (pre + post) for T tokens.
//
// It differentiates L = <dX_out, X'> + <dx_in, x_in> through the forward of include/mhc.h
// ("DeepSeek-V4/mhc": equations rmsnorm, a/b/c-tilde, gate, sinkhorn-init, sinkhorn; the
// slavadubrov.com Eq. 3 read map and merge), the chain rule taken step by step backwards.
// With h the normalised projection the training forward saves, g = alpha * dl the
// gradient of h, r the token's RMS and K = n*d:
//
//   post   dX += H_res^T dX_out, dF_out = H_post^T dX_out,
//          dH_res[i][j] = <dX_out_i, X_j>, dH_post[i] = <dX_out_i, F_out>
//   read   dX += H_pre dx_in, dH_pre[i] = <dx_in, X_i>
//   gates  dl_pre = dH_pre H_pre (1 - H_pre), dl_post = dH_post H_post (1 - H_post / 2)
//   SK     dl_res through the Sinkhorn rounds, recomputed from l_res = alpha_res h_res + b_res
//   proj   dphi += (X_t / r) g^T,   dX_t += phi g / r - X_t (g . h) / (K r^2)
//
// The last term is the RMSNorm backward: sum_k (phi g)_k X_k = r (g . h), so no second
// pass over the channels is needed.
//
// Kernels, in launch order:
//   K1 bwd_reduce   warp per token: the sums over channels (sum X^2, dH_pre, dH_res,
//                   dH_post) into a workspace row, and dF_out
//   K2 bwd_token    thread per token: gates, Sinkhorn backward (each round's input is
//                   kept in shared memory, then the rounds run in reverse), G = g / r and
//                   beta = (g . h) / (K r^2)
//   K3 bwd_dx_dphi  CTA per (channel slice, token group): dX, and the group's partial dphi
//                   (each thread keeps one phi row and one dphi row in registers)
//   K4 reductions   dphi over the groups, db and dalpha over the tokens, all in a fixed
//                   order: repeated runs give bitwise equal results
#include "common.cuh"
#include "launch.cuh"

namespace mhc {
namespace {

constexpr int RED_THREADS = 256;
constexpr int TOK_THREADS = 32;     // K2: one warp per block spreads 16 K tokens over every SM
constexpr int SK_SLOTS = 20;        // K2: Sinkhorn round inputs kept per token
constexpr int DX_THREADS = 256;
constexpr int TB = 32;               // tokens staged per batch in K3
constexpr int UN = 8;                // tokens whose loads K3 has in flight at once
constexpr int SUM_THREADS = 256;

__host__ __device__ constexpr int red_len(int n) { return 1 + n + n * n + n; }

// ---------------------------------------------------------------- K1
// Element pairs of a 16-byte word as float2 (2p, 2p + 1), for the paired FMAs below.
template <typename T> struct Pairs;
template <> struct Pairs<__nv_bfloat16> {
    static constexpr int NP = 4;
    __device__ __forceinline__ static float2 get(const uint4& w, int p) {
        return bf16x2_to_f32x2(p == 0 ? w.x : p == 1 ? w.y : p == 2 ? w.z : w.w);
    }
    // rounds the pair to bf16 into word p
    __device__ __forceinline__ static void put(uint4& w, int p, float2 v) {
        const uint32_t u = pack_bf16x2(v.x, v.y);
        if (p == 0) w.x = u; else if (p == 1) w.y = u; else if (p == 2) w.z = u; else w.w = u;
    }
};
template <> struct Pairs<float> {
    static constexpr int NP = 2;
    __device__ __forceinline__ static float2 get(const uint4& w, int p) {
        return p == 0 ? make_float2(__uint_as_float(w.x), __uint_as_float(w.y))
                      : make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
    }
    __device__ __forceinline__ static void put(uint4& w, int p, float2 v) {
        if (p == 0) { w.x = __float_as_uint(v.x); w.y = __float_as_uint(v.y); }
        else { w.z = __float_as_uint(v.x); w.w = __float_as_uint(v.y); }
    }
};

// One warp per token: the token's reductions R (sum of squares, dx_in . X_i, dX_out_i . X_j,
// dX_out_i . F_out) and dF_out = sum_i H_post[i] dX_out_i.  Each lane walks 16-byte chunks of
// the d channels; its sums run over even and odd channels separately (packed fp32x2 FMAs) and
// are added at the end, then across the warp in a fixed order.
template <int N, typename T>
__global__ void __launch_bounds__(RED_THREADS, 2)
bwd_reduce_kernel(const T* __restrict__ X, const T* __restrict__ F, const T* __restrict__ dY,
                  const T* __restrict__ dx, const float* __restrict__ H, int64_t Tn, int d,
                  float* __restrict__ R, T* __restrict__ dF) {
    constexpr int M = N * N + 2 * N, NR = red_len(N), V = Vec16<T>::VEC;
    using P = Pairs<T>;
    const int lane = threadIdx.x & 31;
    pdl_wait();
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int nchunk = d / V;
    for (int64_t t = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5); t < Tn; t += nwarps) {
        float hpost[N];
#pragma unroll
        for (int i = 0; i < N; ++i) hpost[i] = __ldg(H + t * M + N + N * N + i);
        float2 acc[NR];
#pragma unroll
        for (int q = 0; q < NR; ++q) acc[q] = make_float2(0.f, 0.f);
        for (int q = lane; q < nchunk; q += 32) {
            uint4 wx[N], wy[N];
#pragma unroll
            for (int i = 0; i < N; ++i) wx[i] = ld_stream_v4(X + (t * N + i) * d + q * V);
            const uint4 wd = ld_stream_v4(dx + t * d + q * V);
            const uint4 wf = ld_stream_v4(F + t * d + q * V);
#pragma unroll
            for (int i = 0; i < N; ++i) wy[i] = ld_stream_v4(dY + (t * N + i) * d + q * V);
            uint4 dfw;
#pragma unroll
            for (int p = 0; p < P::NP; ++p) {
                float2 x[N];
#pragma unroll
                for (int i = 0; i < N; ++i) x[i] = P::get(wx[i], p);
                const float2 dv = P::get(wd, p), fv = P::get(wf, p);
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    acc[0] = __ffma2_rn(x[i], x[i], acc[0]);
                    acc[1 + i] = __ffma2_rn(dv, x[i], acc[1 + i]);
                }
                float2 dfp = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    const float2 y = P::get(wy[i], p);
                    acc[1 + N + N * N + i] = __ffma2_rn(y, fv, acc[1 + N + N * N + i]);
                    dfp = __ffma2_rn(make_float2(hpost[i], hpost[i]), y, dfp);
#pragma unroll
                    for (int j = 0; j < N; ++j)
                        acc[1 + N + i * N + j] = __ffma2_rn(y, x[j], acc[1 + N + i * N + j]);
                }
                P::put(dfw, p, dfp);
            }
            st_v4(dF + t * d + q * V, dfw);
        }
        float red[NR];
#pragma unroll
        for (int q = 0; q < NR; ++q) {
            float v = acc[q].x + acc[q].y;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            red[q] = v;
        }
#pragma unroll
        for (int q = 0; q < NR; ++q)
            if (lane == (q & 31)) R[t * NR + q] = red[q];
    }
}

// ---------------------------------------------------------------- K2
// Column then row normalisation of A (one Sinkhorn round); cs, rs receive the reciprocals
// of the column and row sums (fast reciprocals, within 2 ulp: this replay only feeds the
// gradient, whose tolerance is far wider).
template <int N>
__device__ __forceinline__ void sk_round(float (&A)[N][N], float (&B)[N][N], float (&C)[N][N],
                                         float (&cs)[N], float (&rs)[N]) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < N; ++i) s += A[i][j];
        cs[j] = __fdividef(1.0f, s);
#pragma unroll
        for (int i = 0; i < N; ++i) B[i][j] = A[i][j] * cs[j];
    }
#pragma unroll
    for (int i = 0; i < N; ++i) {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < N; ++j) s += B[i][j];
        rs[i] = __fdividef(1.0f, s);
#pragma unroll
        for (int j = 0; j < N; ++j) C[i][j] = B[i][j] * rs[i];
    }
}

template <int N>
__global__ void __launch_bounds__(TOK_THREADS)
bwd_token_kernel(const float* __restrict__ R, const float* __restrict__ H, const float* __restrict__ h,
                 const float* __restrict__ b_res, float a_pre, float a_post, float a_res,
                 int64_t Tn, int K, float eps, int t_max, float* __restrict__ dl,
                 float* __restrict__ G, float* __restrict__ beta, unsigned char* __restrict__ rec) {
    constexpr int M = N * N + 2 * N, NR = red_len(N);
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    pdl_launch_next();          // the dX / dphi step may set itself up meanwhile
    pdl_wait();
    if (t >= Tn) {
        // the tensor-core step's records of the last tile's rows past T are zero
        if (rec != nullptr && t < (Tn + BWD_REC_TILE - 1) / BWD_REC_TILE * BWD_REC_TILE) {
            unsigned char* tile = rec + t / BWD_REC_TILE * (BWD_REC_TILE * BWD_REC_BYTES);
            const int r = (int)(t % BWD_REC_TILE);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                *reinterpret_cast<uint4*>(tile + r * 128 + j * 16) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(tile + 8192 + r * 128 + j * 16) = make_uint4(0, 0, 0, 0);
            }
        }
        return;
    }
    const float* Rt = R + t * NR;
    float hh[M], out[M];
#pragma unroll
    for (int j = 0; j < M; ++j) hh[j] = h[t * M + j];
    // gates
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const float hp = H[t * M + i];
        out[i] = Rt[1 + i] * hp * (1.f - hp);
        const float s = 0.5f * H[t * M + N + N * N + i];
        out[N + N * N + i] = Rt[1 + N + N * N + i] * 2.f * s * (1.f - s);
    }
    // Sinkhorn: M0 = exp(l_res); the backward of round s needs that round's input A_s.
    // The inputs of rounds 0, S, 2S, ... are kept in shared memory (this thread's column of
    // ck), S = 1 while t_max <= SK_SLOTS; A_s is rebuilt by replaying rounds from the kept
    // input at or below s.  That is t_max - 1 + t_max rounds for t_max <= SK_SLOTS instead of
    // the t_max (t_max + 1) / 2 of replaying every A_s from M0.
    __shared__ float ck[SK_SLOTS][N * N][TOK_THREADS];
    const int lane = threadIdx.x;
    float M0[N][N], gM[N][N];
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int j = 0; j < N; ++j) {
            M0[i][j] = expf(a_res * hh[N + i * N + j] + b_res[i * N + j]);
            gM[i][j] = Rt[1 + N + i * N + j];
        }
    // S >= t_max / SK_SLOTS, so every kept index k (k S < t_max) is below SK_SLOTS
    const int S = t_max <= SK_SLOTS ? 1 : (t_max + SK_SLOTS - 1) / SK_SLOTS;
    {
        float A[N][N], B[N][N], C[N][N], cs[N], rs[N];
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int j = 0; j < N; ++j) A[i][j] = M0[i][j];
        for (int k = 0; k * S < t_max; ++k) {
#pragma unroll
            for (int i = 0; i < N; ++i)
#pragma unroll
                for (int j = 0; j < N; ++j) ck[k][i * N + j][lane] = A[i][j];
            if ((k + 1) * S >= t_max) break;
            for (int v = 0; v < S; ++v) {
                sk_round<N>(A, B, C, cs, rs);
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int j = 0; j < N; ++j) A[i][j] = C[i][j];
            }
        }
    }
    for (int s = t_max - 1; s >= 0; --s) {
        float A[N][N], B[N][N], C[N][N], cs[N], rs[N];
        const int k = s / S;
#pragma unroll
        for (int i = 0; i < N; ++i)
#pragma unroll
            for (int j = 0; j < N; ++j) A[i][j] = ck[k][i * N + j][lane];
        for (int u = k * S; u < s; ++u) {
            sk_round<N>(A, B, C, cs, rs);
#pragma unroll
            for (int i = 0; i < N; ++i)
#pragma unroll
                for (int j = 0; j < N; ++j) A[i][j] = C[i][j];
        }
        sk_round<N>(A, B, C, cs, rs);
        // row step C = B / rowsum(B)
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float dot = 0.f;
#pragma unroll
            for (int j = 0; j < N; ++j) dot = fmaf(gM[i][j], C[i][j], dot);
#pragma unroll
            for (int j = 0; j < N; ++j) gM[i][j] = (gM[i][j] - dot) * rs[i];
        }
        // column step B = A / colsum(A)
#pragma unroll
        for (int j = 0; j < N; ++j) {
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < N; ++i) dot = fmaf(gM[i][j], B[i][j], dot);
#pragma unroll
            for (int i = 0; i < N; ++i) gM[i][j] = (gM[i][j] - dot) * cs[j];
        }
    }
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int j = 0; j < N; ++j) out[N + i * N + j] = gM[i][j] * M0[i][j];
    // g = alpha * dl; G = g / r; beta = (g . h) / (K r^2)
    const float inv_r = 1.0f / sqrtf(Rt[0] / (float)K + eps);
    float gh = 0.f, Gv[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
        const float a = j < N ? a_pre : (j < N + N * N ? a_res : a_post);
        const float g = a * out[j];
        gh = fmaf(g, hh[j], gh);
        dl[t * M + j] = out[j];
        Gv[j] = g * inv_r;
    }
    const float bt = gh * inv_r * inv_r / (float)K;
    if (rec == nullptr) {
#pragma unroll
        for (int j = 0; j < M; ++j) G[t * M + j] = Gv[j];
        beta[t] = bt;
        return;
    }
    // the tensor-core step's records (launch.cuh): row r of the token's tile, 16-byte chunk j
    // at position j ^ (r % 8), G row in the first half of the tile, coefficients in the second
    unsigned char* tile = rec + t / BWD_REC_TILE * (BWD_REC_TILE * BWD_REC_BYTES);
    const int r = (int)(t % BWD_REC_TILE);
    auto chunk = [&](int half, int j) {
        return reinterpret_cast<uint4*>(tile + half * 8192 + r * 128 + ((j ^ (r & 7)) << 4));
    };
    uint32_t w[32];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        __nv_bfloat16 hv[2], lv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = 2 * e + u;
            const float v = j < M ? Gv[j] : 0.f;
            hv[u] = __float2bfloat16(v);
            lv[u] = __float2bfloat16(v - __bfloat162float(hv[u]));
        }
        w[e] = (uint32_t)__bfloat16_as_ushort(hv[0]) | ((uint32_t)__bfloat16_as_ushort(hv[1]) << 16);
        w[16 + e] = (uint32_t)__bfloat16_as_ushort(lv[0]) | ((uint32_t)__bfloat16_as_ushort(lv[1]) << 16);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) *chunk(0, j) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float cf[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) cf[q] = 0.f;
        if (i < N) {
            cf[0] = H[t * M + i];
#pragma unroll
            for (int p = 0; p < N; ++p) cf[1 + p] = H[t * M + N + p * N + i];
            cf[5] = -bt;
        }
        *chunk(1, 2 * i) = make_uint4(__float_as_uint(cf[0]), __float_as_uint(cf[1]), __float_as_uint(cf[2]),
                                      __float_as_uint(cf[3]));
        *chunk(1, 2 * i + 1) = make_uint4(__float_as_uint(cf[4]), __float_as_uint(cf[5]), __float_as_uint(cf[6]),
                                          __float_as_uint(cf[7]));
    }
}

// ---------------------------------------------------------------- K3
// Channel slice [c0, c0 + CS) of all N streams: thread (i, c) owns phi row i*d + c.
template <int N, typename T>
__global__ void __launch_bounds__(DX_THREADS)
bwd_dx_dphi_kernel(const T* __restrict__ X, const T* __restrict__ dY, const T* __restrict__ dx,
                   const float* __restrict__ phi, const float* __restrict__ H,
                   const float* __restrict__ G, const float* __restrict__ beta, int64_t Tn, int d,
                   int tpg, T* __restrict__ dX, float* __restrict__ part) {
    constexpr int M = N * N + 2 * N;
    constexpr int CS = DX_THREADS / N >= 256 ? 256 : (DX_THREADS / N >= 128 ? 128 : 64);
    constexpr int MP = (M + 3) / 4 * 4;             // G rows padded for 16-byte reads
    __shared__ __align__(16) float sG[TB][MP];
    __shared__ float sH[TB][M], sB[TB];
    const int i = threadIdx.x / CS;
    const int c = blockIdx.x * CS + (threadIdx.x % CS);
    const bool active = i < N && c < d;
    const int64_t k = (int64_t)i * d + c;
    const int K = N * d;
    float prow[M], acc[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
        prow[j] = active ? __ldg(phi + k * M + j) : 0.f;
        acc[j] = 0.f;
    }
    const int64_t t_lo = (int64_t)blockIdx.y * tpg;
    const int64_t t_hi = t_lo + tpg < Tn ? t_lo + tpg : Tn;
    pdl_wait();
    for (int64_t tb = t_lo; tb < t_hi; tb += TB) {
        const int nb = (int)(t_hi - tb < TB ? t_hi - tb : TB);
        __syncthreads();
        for (int e = threadIdx.x; e < nb * M; e += blockDim.x) {
            const int u = e / M, j = e - u * M;
            sG[u][j] = G[(tb + u) * M + j];
            sH[u][j] = H[(tb + u) * M + j];
        }
        for (int u = threadIdx.x; u < nb; u += blockDim.x) sB[u] = beta[tb + u];
        __syncthreads();
        if (!active) continue;
        // UN tokens at a time: all their loads are issued before any of them is used
        for (int u0 = 0; u0 < nb; u0 += UN) {
            float v[UN], xi[UN], y[UN][N];
#pragma unroll
            for (int q = 0; q < UN; ++q) {
                const int64_t t = tb + (u0 + q < nb ? u0 + q : nb - 1);
                v[q] = to_f32(X[t * K + k]);
                xi[q] = to_f32(dx[t * d + c]);
#pragma unroll
                for (int p = 0; p < N; ++p) y[q][p] = to_f32(dY[t * K + (int64_t)p * d + c]);
            }
#pragma unroll
            for (int q = 0; q < UN; ++q) {
                const int u = u0 + q;
                if (u < nb) {
                    float pg = 0.f;
#pragma unroll
                    for (int j4 = 0; j4 < MP / 4; ++j4) {
                        const float4 g4 = *reinterpret_cast<const float4*>(&sG[u][4 * j4]);
                        const float ge[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = 4 * j4 + e;
                            if (j < M) {
                                acc[j] = fmaf(v[q], ge[e], acc[j]);
                                pg = fmaf(prow[j], ge[e], pg);
                            }
                        }
                    }
                    float g = sH[u][i] * xi[q] + pg - sB[u] * v[q];
#pragma unroll
                    for (int p = 0; p < N; ++p) g = fmaf(sH[u][N + p * N + i], y[q][p], g);
                    store_elem(&dX[(tb + u) * K + k], g);
                }
            }
        }
    }
    if (active) {
        float* p = part + ((int64_t)blockIdx.y * K + k) * M;
#pragma unroll
        for (int j = 0; j < M; ++j) p[j] = acc[j];
    }
}

// ---------------------------------------------------------------- K4
// dphi = sum over the token groups of the partials, in group order.
__global__ void __launch_bounds__(SUM_THREADS)
bwd_dphi_sum_kernel(const float* __restrict__ part, int64_t len, int groups, float* __restrict__ dphi) {
    pdl_wait();
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < len;
         e += (int64_t)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int g = 0; g < groups; ++g) s += part[(int64_t)g * len + e];
        dphi[e] = s;
    }
}

// Column sums over the tokens, in two fixed-order levels.  Partition p (one CTA) covers tokens
// [p * per, (p + 1) * per): thread (u, j), u < CS_ROWS, adds dl[t][j] and dl[t][j] h[t][j] over
// t = start + u, start + u + CS_ROWS, ... (consecutive threads read consecutive floats of a
// row), then the CS_ROWS lanes of a column are added in order into part[p][j], part[p][M + j].
constexpr int CS_PARTS = 64;
template <int M>
__global__ void __launch_bounds__(SUM_THREADS)
bwd_colsum_part_kernel(const float* __restrict__ dl, const float* __restrict__ h, int64_t Tn, int64_t per,
                       float* __restrict__ part) {
    constexpr int CS_ROWS = SUM_THREADS / M;
    __shared__ float s0[CS_ROWS][M], s1[CS_ROWS][M];
    const int u = threadIdx.x / M, j = threadIdx.x % M;
    const int64_t t0 = (int64_t)blockIdx.x * per;
    pdl_wait();
    const int64_t t1 = t0 + per < Tn ? t0 + per : Tn;
    if (u < CS_ROWS) {
        float a = 0.f, b = 0.f;
        for (int64_t t = t0 + u; t < t1; t += CS_ROWS) {
            const float v = dl[t * M + j];
            a += v;
            b = fmaf(v, h[t * M + j], b);
        }
        s0[u][j] = a;
        s1[u][j] = b;
    }
    __syncthreads();
    if (threadIdx.x < M) {
        float a = 0.f, b = 0.f;
#pragma unroll 1
        for (int r = 0; r < CS_ROWS; ++r) {
            a += s0[r][threadIdx.x];
            b += s1[r][threadIdx.x];
        }
        part[(int64_t)blockIdx.x * 2 * M + threadIdx.x] = a;
        part[(int64_t)blockIdx.x * 2 * M + M + threadIdx.x] = b;
    }
}

// The partitions' sums added in partition order; db from the dl sums, dalpha = (pre, post, res)
// sums of the dl * h sums.
template <int N>
__global__ void bwd_colsum_final_kernel(const float* __restrict__ part, int parts, float* __restrict__ db_pre,
                                        float* __restrict__ db_post, float* __restrict__ db_res,
                                        float* __restrict__ dalpha) {
    constexpr int M = N * N + 2 * N;
    __shared__ float cs[2 * M];
    pdl_wait();
    for (int q = threadIdx.x; q < 2 * M; q += blockDim.x) {
        float a = 0.f;
        for (int p = 0; p < parts; ++p) a += part[(int64_t)p * 2 * M + q];
        cs[q] = a;
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    float ap = 0.f, ar = 0.f, aq = 0.f;
    for (int j = 0; j < N; ++j) { db_pre[j] = cs[j]; ap += cs[M + j]; }
    for (int q = 0; q < N * N; ++q) { db_res[q] = cs[N + q]; ar += cs[M + N + q]; }
    for (int j = 0; j < N; ++j) { db_post[j] = cs[N + N * N + j]; aq += cs[M + N + N * N + j]; }
    dalpha[0] = ap;
    dalpha[1] = aq;
    dalpha[2] = ar;
}

int dx_slice(int n) { return DX_THREADS / n >= 256 ? 256 : (DX_THREADS / n >= 128 ? 128 : 64); }

template <int N, typename T>
cudaError_t launch_n(const BwdArgs& a, const BwdLayout& L) {
    constexpr int M = N * N + 2 * N;
    const int64_t Tn = a.T;
    const int d = a.d, K = N * d;
    const T* X = static_cast<const T*>(a.X);
    const T* dY = static_cast<const T*>(a.dX_out);
    const T* dxi = static_cast<const T*>(a.dx_in);
    float* ws = static_cast<float*>(a.workspace);
    float* R = ws + L.off_R;
    float* dl = ws + L.off_dl;
    float* G = ws + L.off_G;
    float* beta = ws + L.off_beta;
    float* part = ws + L.off_part;
    float* colsum = ws + L.off_colsum;
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    {
        int64_t blocks = (Tn * 32 + RED_THREADS - 1) / RED_THREADS;
        const int64_t cap = (int64_t)di.sm_count * 8;
        if (blocks > cap) blocks = cap;
        e = launch_pdl(bwd_reduce_kernel<N, T>, dim3((unsigned)blocks), dim3(RED_THREADS), 0, a.stream, X,
                       static_cast<const T*>(a.F), dY, dxi, a.H, Tn, d, R, static_cast<T*>(a.dF_out));
        if (e != cudaSuccess) return e;
    }
    unsigned char* rec = L.tc ? reinterpret_cast<unsigned char*>(ws + L.off_rec) : nullptr;
    const int64_t tok_threads = L.tc ? (Tn + BWD_REC_TILE - 1) / BWD_REC_TILE * BWD_REC_TILE : Tn;
    e = launch_pdl(bwd_token_kernel<N>, dim3((unsigned)((tok_threads + TOK_THREADS - 1) / TOK_THREADS)),
                   dim3(TOK_THREADS), 0, a.stream, (const float*)R, a.H, a.h, a.b_res, a.a_pre, a.a_post, a.a_res,
                   Tn, K, a.eps, a.t_max, dl, G, beta, rec);
    if (e != cudaSuccess) return e;
    if (L.tc) {
        e = launch_bwd_tc(a, rec, part, L.groups, L.tokens_per_group);
        if (e != cudaSuccess) return e;
    } else {
        const int cs = dx_slice(N);
        dim3 grid((unsigned)((d + cs - 1) / cs), (unsigned)L.groups);
        e = launch_pdl(bwd_dx_dphi_kernel<N, T>, grid, dim3(DX_THREADS), 0, a.stream, X, dY, dxi, a.phi, a.H,
                       (const float*)G, (const float*)beta, Tn, d, (int)L.tokens_per_group, static_cast<T*>(a.dX),
                       part);
        if (e != cudaSuccess) return e;
    }
    {
        const int64_t len = (int64_t)K * M;
        int64_t blocks = (len + SUM_THREADS - 1) / SUM_THREADS;
        if (blocks > (int64_t)di.sm_count * 8) blocks = (int64_t)di.sm_count * 8;
        e = launch_pdl(bwd_dphi_sum_kernel, dim3((unsigned)blocks), dim3(SUM_THREADS), 0, a.stream,
                       (const float*)part, len, L.groups, a.dphi);
        if (e != cudaSuccess) return e;
    }
    {
        const int64_t per = (Tn + CS_PARTS - 1) / CS_PARTS;
        e = launch_pdl(bwd_colsum_part_kernel<M>, dim3(CS_PARTS), dim3(SUM_THREADS), 0, a.stream,
                       (const float*)dl, a.h, Tn, per, colsum);
        if (e != cudaSuccess) return e;
        e = launch_pdl(bwd_colsum_final_kernel<N>, dim3(1), dim3(64), 0, a.stream, (const float*)colsum,
                       (int)CS_PARTS, a.db_pre, a.db_post, a.db_res, a.dalpha);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch(const BwdArgs& a, const BwdLayout& L) {
    switch (a.n) {
        case 1: return launch_n<1, T>(a, L);
        case 2: return launch_n<2, T>(a, L);
        case 3: return launch_n<3, T>(a, L);
        case 4: return launch_n<4, T>(a, L);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

BwdLayout backward_layout(int64_t T, int n, int d, bool tc) {
    BwdLayout L{};
    const int64_t m = (int64_t)n * n + 2 * n, K = (int64_t)n * d;
    L.tc = tc && d % 64 == 0 && d >= 64;
    if (L.tc) {
        L.groups = bwd_tc_groups(T, d, BWD_TC_SMS);
        L.tokens_per_group = bwd_tc_tokens_per_group(T, L.groups);
    } else {
        const int64_t slices = (d + dx_slice(n) - 1) / dx_slice(n);
        // about 1024 CTAs in K3, each group at least 32 tokens
        int64_t groups = (1024 + slices - 1) / slices;
        const int64_t max_groups = (T + TB - 1) / TB;
        if (groups > max_groups) groups = max_groups;
        if (groups < 1) groups = 1;
        L.groups = (int)groups;
        L.tokens_per_group = (T + groups - 1) / groups;
    }
    auto up = [](int64_t x) { return (x + 63) / 64 * 64; };   // 256-byte aligned regions
    int64_t off = 0;
    L.off_R = off;      off += up(T * red_len(n));
    L.off_dl = off;     off += up(T * m);
    if (L.tc) {
        L.off_rec = off; off += up((T + BWD_REC_TILE - 1) / BWD_REC_TILE * BWD_REC_TILE * (BWD_REC_BYTES / 4));
    } else {
        L.off_G = off;      off += up(T * m);
        L.off_beta = off;   off += up(T);
    }
    L.off_part = off;   off += up((int64_t)L.groups * K * m);
    L.off_colsum = off; off += up(CS_PARTS * 2 * m);   // the column sums' partitions
    L.floats = off;
    return L;
}

int64_t backward_workspace_floats(int64_t T, int n, int d) {
    const int64_t a = backward_layout(T, n, d, false).floats, b = backward_layout(T, n, d, true).floats;
    return a > b ? a : b;
}

cudaError_t launch_backward(const BwdArgs& a) {
    const bool tc = bwd_tc_shape_ok(a.T, a.n, a.d, a.dt) && bwd_tc_device_ok(a.n);
    const BwdLayout L = backward_layout(a.T, a.n, a.d, tc);
    return a.dt == BF16 ? dispatch<__nv_bfloat16>(a, L) : dispatch<float>(a, L);
}

}  // namespace mhc
