// backward_tc.cu -- the dX / dphi step of the mHC backward on sm_100a tensor cores.
//
// With G_t = g_t / r_t (the gradient of the token's normalised projection h_t, over its RMS)
// and beta_t = (g_t . h_t) / (K r_t^2) from the token kernel (backward.cu), the step computes
// for token t and flattened channel k = i d + c ("DeepSeek-V4/mhc" equation rmsnorm and the
// slavadubrov.com Eq. 3 read map and merge, differentiated):
//
//   dX[t][i][c] = H_pre[i] dx_in[t][c] + sum_p H_res[p][i] dX_out[t][p][c]
//                 + (phi G_t)[k] - beta_t X[t][i][c]
//   dphi[k][j]  = sum_t X[t][k] G_t[j]
//
// Both products are thin (one side is m = n^2 + 2n wide).  On tcgen05:
//   * CTA (s, g) owns channels [64 s, 64 s + 64) of every stream and the tokens of group g.
//     Its MMA rows are k: block b holds stream 2b in rows 0-63 and stream 2b + 1 in rows
//     64-127 (for odd n the last block's upper half is a placeholder whose rows are unused).
//   * phi G: A = the CTA's rows of phi, resident in TMEM as bf16 with K = 96,
//     [phi_hi | phi_hi | phi_lo]; B = the token's record [G_hi | G_lo | G_hi], K-major in
//     shared memory.  The sum is phi G less the phi_lo G_lo term: 16 significant bits on
//     both sides.  D[k][t] (M = 128, N = 64 tokens) lands in TMEM, two buffers deep.
//   * dphi: A = X^T, read by the tensor core straight from the stage's TMA tile (MN-major:
//     64 channels in each 128-byte row, tokens down the rows); B = [G_hi | G_lo] from the
//     same records (MN-major).  D[k][j] accumulates in TMEM over all of the group's tokens.
//   * Eight warps form dX.  TMEM lane = row k, so a thread owns channel c of two streams; it
//     walks the stage's tokens, reading X, dX_out and dx_in from shared memory and the
//     token's coefficients (H_pre[i], H_res[.][i], -beta) from the record.
//
// A stage is 64 tokens: TMA boxes of the CTA's slice of X and dX_out (64 channels x 64
// tokens x n streams), of dx_in (64 x 64) and of the 64 token records (384 B each).
// Warp roles (320 threads): 0 TMA producer, 1 TMEM owner and MMA issuer, 2-9 phi into TMEM
// at the start, the dX epilogue, the dphi partials at the end.  Every wait on an mbarrier is
// bounded in time; on expiry the kernel records the wait in a status word and returns
// after its copies and MMAs in flight have completed.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.cuh"
#include "tc_ptx.cuh"

namespace mhc {

// Status of the tensor-core backward kernel's bounded waits since the last read: 0 = fine,
// otherwise an OR of the codes of the waits that expired (mhc_device_status).
__device__ unsigned int g_bwd_tc_status;

namespace bwdtc {

constexpr int TT = 64;                 // tokens per stage = N of the phi G product
constexpr int CW = 64;                 // channels of a CTA's slice (one 128-byte row)
constexpr int ROW = 128;               // bytes per row of a tile
constexpr int NBUF = 2;                // phi G accumulator buffers
constexpr int EPI = 8;                 // epilogue warps: two per TMEM lane quarter
constexpr int THREADS = 32 * (2 + EPI);
constexpr int KP16 = 6;                // K16 steps of phi G (K = 96)
constexpr int SMEM_STAGES_MAX = 200 * 1024;
constexpr unsigned long long kWaitNs = 1000000000ull;    // 1 s per wait
constexpr unsigned long long kDrainNs = 2000000000ull;   // 2 s for the drains at exit

template <int N>
struct Cfg {
    static constexpr int M = N * N + 2 * N;
    static constexpr int NB = (N + 1) / 2;                 // MMA row blocks of 128
    static constexpr int XB = N * TT * ROW;                // X or dX_out box
    static constexpr int DXB = TT * ROW;                   // dx_in box
    static constexpr int GB = 3 * TT * ROW;                // token records box
    static constexpr int STAGE = 2 * XB + DXB + GB;
    static constexpr int NS = SMEM_STAGES_MAX / STAGE > 4 ? 4 : SMEM_STAGES_MAX / STAGE;
    static constexpr int SMEM = NS * STAGE + 1024;         // + alignment slack
    static constexpr int PG_COL = 0;                       // [buf][b]: TT columns each
    static constexpr int DPHI_COL = NBUF * NB * TT;        // [b]: 64 columns each
    static constexpr int A_COL = DPHI_COL + NB * 64;       // [b]: 48 columns each
    static constexpr int COLS = A_COL + NB * 48;
    static constexpr int TMEM_COLS = COLS <= 256 ? 256 : 512;
    static_assert(M <= 32, "G_hi, G_lo fit 32 columns each");
    static_assert(NS >= 2, "at least two stages");
    static_assert(COLS <= 512, "TMEM columns");
    static_assert(N <= 4, "coefficients of at most 4 streams per record");
};

// instruction descriptor, kind::f16: D fp32, A and B bf16, M = 128, N = nb
__host__ __device__ constexpr uint32_t idesc(int nb, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(nb >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

enum : unsigned { E_EMPTY = 1u, E_FULL = 2u, E_PGEMPTY = 4u, E_PGFULL = 8u, E_DRAIN = 16u };

using namespace ptx;

struct Waiter {
    volatile int* abort_flag;
    unsigned long long limit_ns;
    // true when the phase completed; false when the CTA is aborting or the wait expired
    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity, unsigned code,
                                               bool honour_abort = true) const {
        if (mbar_try(bar, parity)) return true;
        const uint64_t t0 = gtimer();
        while (true) {
            if (mbar_try(bar, parity)) return true;
            if (honour_abort && *abort_flag) return false;
            if (gtimer() - t0 > limit_ns) {
                atomicOr(&g_bwd_tc_status, code);
                *abort_flag = 1;
                return false;
            }
        }
    }
};

__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr) : "memory");
}
// wait for this thread's TMEM loads; the registers are operands, so no use of them is
// scheduled before the wait
__device__ __forceinline__ void tmem_wait16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                   "+r"(r[13]), "+r"(r[14]), "+r"(r[15]) :: "memory");
}
__device__ __forceinline__ float ld_bf16(const unsigned char* p) {
    return __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(p)) << 16);
}
__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

struct Maps {
    CUtensorMap x;      // X viewed as (c: d, t: T, i: n), box (64, TT, n)
    CUtensorMap dy;     // dX_out, the same view
    CUtensorMap dx;     // dx_in (c: d, t: T), box (64, TT)
    CUtensorMap rec;    // token records (e: 64, t: T, row: 3), box (64, TT, 3)
};

enum : int { B_FULL = 0, B_EMPTY = 4, B_PGF = 8, B_PGE = 10, B_COUNT = 12 };

template <int N>
__global__ void __launch_bounds__(THREADS, 1)
bwd_tc_kernel(const __grid_constant__ Maps maps, const float* __restrict__ phi, int T, int d, int tpg,
              __nv_bfloat16* __restrict__ dX, float* __restrict__ part) {
    using C = Cfg<N>;
    constexpr int M = C::M, NB = C::NB, NS = C::NS;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t bars[B_COUNT];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    const Waiter wait{&abort_flag, kWaitNs};
    const Waiter drain{&abort_flag, kDrainNs};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slices = d / CW;
    const int s = (int)(blockIdx.x % (unsigned)slices), g = (int)(blockIdx.x / (unsigned)slices);
    const int c0 = s * CW;
    const int64_t t_lo64 = (int64_t)g * tpg;
    const int t_lo = (int)(t_lo64 < T ? t_lo64 : T);
    const int t_hi = (int)(t_lo64 + tpg < T ? t_lo64 + tpg : T);
    const int nst = (t_hi - t_lo + TT - 1) / TT;
    const int K = N * d;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(bar(B_FULL + i), 1);
            mbar_init(bar(B_EMPTY + i), EPI);
        }
        for (int i = 0; i < NBUF; ++i) {
            mbar_init(bar(B_PGF + i), 1);
            mbar_init(bar(B_PGE + i), EPI);
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_slot;

    // phi rows into TMEM: epilogue warp (quarter q, half b) writes row 32 q + lane of block b
    if (warp >= 2) {
        const int q = warp & 3, b = (warp - 2) >> 2;
        if (b < NB) {
            const int i = 2 * b + (q >> 1), c = 32 * (q & 1) + lane;
            __nv_bfloat16 hi[32], lo[32];
            const __nv_bfloat16 z = __float2bfloat16(0.f);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float v = (j < M && i < N) ? __ldg(phi + ((int64_t)i * d + c0 + c) * M + j) : 0.f;
                hi[j] = __float2bfloat16(v);
                lo[j] = j < M ? __float2bfloat16(v - __bfloat162float(hi[j])) : z;
            }
            uint4 w[12];
            uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
            for (int e = 0; e < 16; ++e) {            // K 0..31: hi; 32..63: hi; 64..95: lo
                wp[e] = pack_bf16x2(hi[2 * e], hi[2 * e + 1]);
                wp[16 + e] = wp[e];
                wp[32 + e] = pack_bf16x2(lo[2 * e], lo[2 * e + 1]);
            }
            const uint32_t ta = tm + ((uint32_t)(32 * q) << 16) + C::A_COL + 48 * b;
            tmem_st16(ta, *reinterpret_cast<const uint4(*)[4]>(&w[0]));
            tmem_st16(ta + 16, *reinterpret_cast<const uint4(*)[4]>(&w[4]));
            tmem_st16(ta + 32, *reinterpret_cast<const uint4(*)[4]>(&w[8]));
            tmem_wait_st();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < nst; ++it) {
                const int st = it % NS;
                if (it >= NS && !wait(bar(B_EMPTY + st), (uint32_t)((it / NS) - 1) & 1u, E_EMPTY)) break;
                const uint32_t base = smem_u32(sm + st * C::STAGE);
                const uint32_t full = bar(B_FULL + st);
                const int t0 = t_lo + it * TT;
                mbar_arrive_tx(full, (uint32_t)C::STAGE);
                tma_load_3d(base, &maps.x, full, c0, t0, 0);
                tma_load_3d(base + C::XB, &maps.dy, full, c0, t0, 0);
                tma_load_2d(base + 2 * C::XB, &maps.dx, full, c0, t0);
                tma_load_3d(base + 2 * C::XB + C::DXB, &maps.rec, full, 0, t0, 0);
                issued = it + 1;
            }
            // the copies of the last stages must have landed before the CTA exits
            for (int it = issued - NS > 0 ? issued - NS : 0; it < issued; ++it)
                drain(bar(B_FULL + it % NS), (uint32_t)(it / NS) & 1u, E_DRAIN, false);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_DPHI = idesc(64, 1, 1);   // A = X^T, B = [G_hi | G_lo], both MN-major
            constexpr uint32_t ID_PG = idesc(TT, 0, 0);     // A = phi (TMEM), B = records, K-major
            int done = 0;
            for (int it = 0; it < nst; ++it) {
                const int st = it % NS, buf = it & 1;
                if (!wait(bar(B_FULL + st), (uint32_t)(it / NS) & 1u, E_FULL)) break;
                if (it >= NBUF && !wait(bar(B_PGE + buf), (uint32_t)((it >> 1) - 1) & 1u, E_PGEMPTY)) break;
                tc_fence_after();
                const uint32_t xs = smem_u32(sm + st * C::STAGE);
                const uint32_t gs = xs + 2 * C::XB + C::DXB;
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int k = 0; k < TT / 16; ++k)
                        mma_bf16(tm + C::DPHI_COL + 64 * b,
                                 sw128_desc_mn(xs + 2 * b * TT * ROW + k * 2048, TT * ROW, 1024),
                                 sw128_desc_mn(gs + k * 2048, TT * ROW, 1024), ID_DPHI,
                                 (it > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int k = 0; k < KP16; ++k)
                        mma_bf16_tmem_a(tm + C::PG_COL + (buf * NB + b) * TT, tm + C::A_COL + 48 * b + 8 * k,
                                        sw128_desc(gs + (k >> 2) * TT * ROW + (k & 3) * 32), ID_PG,
                                        k > 0 ? 1u : 0u);
                mma_commit(bar(B_PGF + buf));
                done = it + 1;
            }
            // TMEM must be idle before it is freed
            if (done > 0) drain(bar(B_PGF + ((done - 1) & 1)), (uint32_t)((done - 1) >> 1) & 1u, E_DRAIN, false);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- dX epilogue
        const int q = warp & 3, h = (warp - 2) >> 2;
        const int ih = q >> 1, c = 32 * (q & 1) + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        bool ok = true;
        for (int it = 0; it < nst; ++it) {
            const int st = it % NS, buf = it & 1;
            if (!wait(bar(B_FULL + st), (uint32_t)(it / NS) & 1u, E_FULL) ||
                !wait(bar(B_PGF + buf), (uint32_t)(it >> 1) & 1u, E_PGFULL)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const unsigned char* xs = sm + st * C::STAGE;
            const unsigned char* ys = xs + C::XB;
            const unsigned char* ds = xs + 2 * C::XB;
            const unsigned char* cs = ds + C::DXB + 2 * TT * ROW;     // record row 2: coefficients
            const int t0 = t_lo + it * TT;
#pragma unroll 1
            for (int ch = 0; ch < 2; ++ch) {
                const int col = h * 32 + ch * 16;
                uint32_t pg[NB][16];
#pragma unroll
                for (int b = 0; b < NB; ++b) tmem_ld16_nowait(tm + lane_base + C::PG_COL + (buf * NB + b) * TT + col, pg[b]);
#pragma unroll
                for (int b = 0; b < NB; ++b) tmem_wait16(pg[b]);
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int tl = col + u;
                    const int t = t0 + tl;
                    const uint32_t roff = sw128_off(tl, c >> 3) + (c & 7) * 2;
                    const float dxv = ld_bf16(ds + roff);
                    float dy[N];
#pragma unroll
                    for (int p = 0; p < N; ++p) dy[p] = ld_bf16(ys + p * TT * ROW + roff);
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const int i = 2 * b + ih;
                        if (i < N) {
                            const float4 ca = *reinterpret_cast<const float4*>(cs + sw128_off(tl, 2 * i));
                            const float4 cb = *reinterpret_cast<const float4*>(cs + sw128_off(tl, 2 * i + 1));
                            const float cr[4] = {ca.y, ca.z, ca.w, cb.x};
                            const float xv = ld_bf16(xs + i * TT * ROW + roff);
                            float v = fmaf(ca.x, dxv, __uint_as_float(pg[b][u]));
                            v = fmaf(cb.y, xv, v);
#pragma unroll
                            for (int p = 0; p < N; ++p) v = fmaf(cr[p], dy[p], v);
                            if (t < t_hi) dX[((int64_t)t * N + i) * d + c0 + c] = __float2bfloat16(v);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_PGE + buf));
                mbar_arrive(bar(B_EMPTY + st));
            }
        }
        // dphi partials of the group: warp half h reads block h (its last phi G wait covered
        // every MMA of the CTA)
        const int b = h;
        if (ok && b < NB) {
            const int i = 2 * b + ih;
            if (i < N) {
                float* dst = part + ((int64_t)g * K + (int64_t)i * d + c0 + c) * M;
                if (nst > 0) {
                    float vh[32], vl[32];
                    tmem_ld32(tm + lane_base + C::DPHI_COL + 64 * b, vh);
                    tmem_ld32(tm + lane_base + C::DPHI_COL + 64 * b + 32, vl);
#pragma unroll
                    for (int j = 0; j < M; ++j) dst[j] = vh[j] + vl[j];
                } else {
#pragma unroll
                    for (int j = 0; j < M; ++j) dst[j] = 0.f;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, C::TMEM_COLS);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        cudaGetLastError();
    });
    return fn;
}

template <int N>
bool configure() {
    static int ok = -1;
    if (ok < 0) {
        ok = cudaFuncSetAttribute(bwd_tc_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<N>::SMEM) ==
             cudaSuccess;
        cudaGetLastError();
    }
    return ok == 1;
}

template <int N>
cudaError_t launch_n(const BwdArgs& a, const void* rec, float* part, int groups, int64_t tpg) {
    auto enc = encode_fn();
    if (!enc || !configure<N>()) return cudaErrorNotSupported;
    Maps maps;
    const cuuint32_t e1[3] = {1, 1, 1};
    CUresult r;
    {   // X and dX_out: dims (c, t, i), strides t: n d, i: d elements
        const cuuint64_t dims[3] = {(cuuint64_t)a.d, (cuuint64_t)a.T, (cuuint64_t)N};
        const cuuint64_t str[2] = {(cuuint64_t)N * a.d * 2, (cuuint64_t)a.d * 2};
        const cuuint32_t box[3] = {CW, TT, N};
        r = enc(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.X), dims, str, box, e1,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        r = enc(&maps.dy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.dX_out), dims, str, box, e1,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    {   // dx_in: dims (c, t)
        const cuuint64_t dims[2] = {(cuuint64_t)a.d, (cuuint64_t)a.T};
        const cuuint64_t str[1] = {(cuuint64_t)a.d * 2};
        const cuuint32_t box[2] = {CW, TT};
        r = enc(&maps.dx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.dx_in), dims, str, box, e1,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    {   // records: dims (e, t, row), strides t: 384 B, row: 128 B
        const cuuint64_t dims[3] = {64, (cuuint64_t)a.T, 3};
        const cuuint64_t str[2] = {(cuuint64_t)BWD_REC_BYTES, 128};
        const cuuint32_t box[3] = {64, TT, 3};
        r = enc(&maps.rec, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(rec), dims, str, box, e1,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    const int slices = a.d / CW;
    const unsigned grid = (unsigned)(slices * groups);
    bwd_tc_kernel<N><<<grid, THREADS, Cfg<N>::SMEM, a.stream>>>(maps, a.phi, (int)a.T, a.d, (int)tpg,
                                                                static_cast<__nv_bfloat16*>(a.dX), part);
    return cudaGetLastError();
}

}  // namespace bwdtc

bool bwd_tc_shape_ok(int64_t T, int n, int d, DType dt) {
    return dt == BF16 && n >= 1 && n <= 4 && d >= bwdtc::CW && d % bwdtc::CW == 0 && T >= 1 &&
           T < ((int64_t)1 << 31) - 2 * bwdtc::TT;
}

bool bwd_tc_device_ok(int n) {
    switch (n) {
        case 1: return bwdtc::configure<1>();
        case 2: return bwdtc::configure<2>();
        case 3: return bwdtc::configure<3>();
        case 4: return bwdtc::configure<4>();
        default: return false;
    }
}

int bwd_tc_groups(int64_t T, int d, int sm_count) {
    const int slices = d / bwdtc::CW;
    int64_t g = slices >= sm_count ? 1 : sm_count / slices;
    const int64_t stages = (T + bwdtc::TT - 1) / bwdtc::TT;
    if (g > stages) g = stages;
    return g < 1 ? 1 : (int)g;
}

int64_t bwd_tc_tokens_per_group(int64_t T, int groups) {
    const int64_t per = (T + groups - 1) / groups;
    return (per + bwdtc::TT - 1) / bwdtc::TT * bwdtc::TT;
}

cudaError_t launch_bwd_tc(const BwdArgs& a, const void* rec, float* part, int groups, int64_t tpg) {
    switch (a.n) {
        case 1: return bwdtc::launch_n<1>(a, rec, part, groups, tpg);
        case 2: return bwdtc::launch_n<2>(a, rec, part, groups, tpg);
        case 3: return bwdtc::launch_n<3>(a, rec, part, groups, tpg);
        case 4: return bwdtc::launch_n<4>(a, rec, part, groups, tpg);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t bwd_tc_status(unsigned* out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_bwd_tc_status, sizeof(unsigned));
    if (e != cudaSuccess) return e;
    if (clear && *out) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_bwd_tc_status, &zero, sizeof(unsigned));
    }
    return e;
}

}  // namespace mhc
