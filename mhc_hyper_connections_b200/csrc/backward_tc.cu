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
//   * CTA (s, g) owns channels [64 s, 64 s + 64) of every stream and the tokens of group g:
//     k rows 0-63 are stream 0 of the slice, 64-127 stream 1, and so on (for odd n a
//     placeholder stream fills the last 64 rows; its results are not used).
//   * phi G as D[t][k]: A = G_t as bf16 [G_hi | G_lo] (the token's record row), B = the CTA's
//     rows of phi, resident in shared memory as [phi_hi | phi_lo]; three products of K = 32
//     (G_hi phi_hi, G_lo phi_hi, G_hi phi_lo), taken by pointing the descriptors at the halves
//     of the rows: phi G less the phi_lo G_lo term, 16 significant bits on both sides.  A
//     stage's 64 tokens are M: streams 0-1 go to one M = 64 accumulator in TMEM lanes 0-15 of
//     each lane quarter, streams 2-3 to a second in lanes 16-31, so every lane of a TMEM load
//     holds a token.
//   * dphi: A = X^T, read by the tensor core straight from the stage's TMA tile (MN-major:
//     64 channels in each 128-byte row, tokens down the rows); B = [G_hi | G_lo] from the
//     same rows (MN-major).  D[k][j] (M = 128: two streams) accumulates in TMEM over all
//     of the group's tokens.
//   * Eight warps form dX: a thread owns a token, two streams and 32 channels; it reads X,
//     dX_out and dx_in from the stage in 16-byte vectors and its token's coefficients
//     (H_pre[i], H_res[.][i], -beta) from the stage's record tile, and writes dX over the dX_out
//     rows it has consumed; one TMA store per stage writes the tile.
//
// A stage is 64 tokens: one bulk copy of the 64 tokens' records (G rows and coefficients,
// swizzled by the token kernel; on their own barrier, so phi G runs while the rest lands) and
// TMA boxes of the CTA's slice of X and dX_out (64 channels x 64 tokens x n streams) and of
// dx_in (64 x 64).  The dphi MMAs are issued after phi G.  A slot is reloaded once its dX tile
// has been stored and its dphi MMAs have completed.
// Warp roles (320 threads): 0 TMA loads and stores, 1 TMEM owner and MMA issuer, 2-9 phi into
// shared memory at the start, the dX epilogue, the dphi partials at the end.  Every wait on an
// mbarrier is bounded in time; on expiry the kernel records the wait in a status word and
// returns after its copies and MMAs in flight have completed.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "launch.cuh"
#include "tc_ptx.cuh"

namespace mhc {

// Status of the tensor-core backward kernel's bounded waits since the last read: 0 = fine,
// otherwise an OR of the codes of the waits that expired (mhc_device_status).
__device__ unsigned int g_bwd_tc_status;

namespace bwdtc {

constexpr int TT = 64;                 // tokens per stage = M of the phi G product
constexpr int CW = 64;                 // channels of a CTA's slice (one 128-byte row)
constexpr int ROW = 128;               // bytes per row of a tile
constexpr int NBUF = 2;                // phi G accumulator buffers
constexpr int PGN = 128;               // N of one phi G MMA: two streams of the slice
constexpr int EPI = 8;                 // epilogue warps: two per TMEM lane quarter, 32 channels each
constexpr int THREADS = 32 * (2 + EPI);
constexpr int KP16 = 6;                // K16 steps of phi G (K = 96)
constexpr int SMEM_LIMIT = 232448 - 512;   // dynamic shared memory, less the static part
constexpr unsigned long long kWaitNs = 1000000000ull;    // 1 s per wait
constexpr unsigned long long kDrainNs = 2000000000ull;   // 2 s for the drains at exit
constexpr uint32_t kSuspendNs = 20000;  // a waiting thread sleeps up to this long per try

template <int N>
struct Cfg {
    static constexpr int M = N * N + 2 * N;
    static constexpr int NB = (N + 1) / 2;                 // stream pairs (dphi blocks, phi G halves)
    static constexpr int NR = NB * PGN;                    // k rows of phi, placeholder rows included
    static constexpr int PHI = NR * ROW;                   // one [phi_hi | phi_lo] row per k
    static constexpr int XB = N * TT * ROW;                // X or dX_out box
    static constexpr int DXB = TT * ROW;                   // dx_in box
    static constexpr int GB = BWD_REC_TILE * BWD_REC_BYTES;   // the stage's record tile: G rows, coefficients
    static constexpr int STAGE = 2 * XB + DXB + GB;
    static constexpr int NS_FIT = (SMEM_LIMIT - 1024 - PHI) / STAGE;
    static constexpr int NS = NS_FIT > 4 ? 4 : NS_FIT;
    static constexpr int SMEM = NS * STAGE + PHI + 1024;   // + alignment slack
    static constexpr int PG_COL = 0;                       // [buf]: PGN columns, lane base 16 per half
    static constexpr int DPHI_COL = NBUF * PGN;            // [b]: 64 columns each
    static constexpr int COLS = DPHI_COL + NB * 64;
    static constexpr int TMEM_COLS = COLS <= 256 ? 256 : 512;
    static_assert(M <= 32, "G_hi, G_lo fit 32 columns each");
    static_assert(NS >= 2, "at least two stages");
    static_assert(SMEM <= SMEM_LIMIT, "shared memory");
    static_assert(COLS <= 512, "TMEM columns");
    static_assert(N <= 4, "coefficients of at most 4 streams per record");
};

// instruction descriptor, kind::f16: D fp32, A and B bf16, M = mm, N = nb
__host__ __device__ constexpr uint32_t idesc(int mm, int nb, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(nb >> 3) << 17) | ((uint32_t)(mm >> 4) << 24);
}

enum : unsigned { E_EMPTY = 1u, E_FULL = 2u, E_PGEMPTY = 4u, E_PGFULL = 8u, E_DRAIN = 16u };

using namespace ptx;

// try_wait that may suspend the thread until the phase completes or `ns` pass
__device__ __forceinline__ bool mbar_try_sleep(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "r"(ns) : "memory");
    return ok != 0;
}

struct Waiter {
    volatile int* abort_flag;
    unsigned long long limit_ns;
    // true when the phase completed; false when the CTA is aborting or the wait expired
    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity, unsigned code,
                                               bool honour_abort = true) const {
        if (mbar_try(bar, parity)) return true;
        const uint64_t t0 = gtimer();
        while (true) {
            if (mbar_try_sleep(bar, parity, kSuspendNs)) return true;
            if (honour_abort && *abort_flag) return false;
            if (gtimer() - t0 > limit_ns) {
                atomicOr(&g_bwd_tc_status, code);
                *abort_flag = 1;
                return false;
            }
        }
    }
};

template <int W>
__device__ __forceinline__ void tmem_ld_x(uint32_t taddr, uint32_t (&r)[W]);
template <>
__device__ __forceinline__ void tmem_ld_x<32>(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
                   "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
                   "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
                   "=r"(r[31])
                 : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_x<8>(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_wait8(uint32_t (&r)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]) :: "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_x<16>(uint32_t taddr, uint32_t (&r)[16]) {
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
__device__ __forceinline__ void tmem_wait32(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                   "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
                   "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
                   "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
                   "+r"(r[31]) :: "memory");
}
// bf16 pair (low, high halves of a word) to two floats
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}
__device__ __forceinline__ uint32_t pack_f32x2(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}

struct Maps {
    CUtensorMap x;      // X viewed as (c: d, t: T, i: n), box (64, TT, n)
    CUtensorMap dy;     // dX_out, the same view
    CUtensorMap dx;     // dx_in (c: d, t: T), box (64, TT)
    CUtensorMap dxo;    // dX, the view of X (stores)
};

// FULLG: the stage's record tile landed; FULL: its X, dX_out, dx_in landed; EPID: the epilogue has
// written the stage's dX tile; DPHID: the stage's dphi MMAs are done; PGF / PGE: phi G accumulator
// full / free; MMAD: every MMA of the CTA has completed
enum : int {
    B_FULLG = 0, B_FULL = 4, B_EPID = 8, B_DPHID = 12, B_PGF = 16, B_PGE = 18, B_MMAD = 20, B_COUNT = 21
};

template <int N>
__global__ void __launch_bounds__(THREADS, 1)
bwd_tc_kernel(const __grid_constant__ Maps maps, const float* __restrict__ phi,
              const unsigned char* __restrict__ rec, int T, int d, int tpg, __nv_bfloat16* __restrict__ dX,
              float* __restrict__ part, int stop_stage, unsigned long long wait_ns) {
    using C = Cfg<N>;
    constexpr int M = C::M, NB = C::NB, NS = C::NS;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    unsigned char* phs = sm + NS * C::STAGE;          // phi rows [phi_hi | phi_lo]
    __shared__ __align__(8) uint64_t bars[B_COUNT];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    const Waiter wait{&abort_flag, wait_ns};
    const Waiter drain{&abort_flag, wait_ns > kDrainNs ? wait_ns : kDrainNs};   // drains keep their full limit

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
            mbar_init(bar(B_FULLG + i), 1);
            mbar_init(bar(B_FULL + i), 1);
            mbar_init(bar(B_EPID + i), EPI);
            mbar_init(bar(B_DPHID + i), 1);
        }
        mbar_init(bar(B_MMAD), 1);
        for (int i = 0; i < NBUF; ++i) {
            mbar_init(bar(B_PGF + i), 1);
            mbar_init(bar(B_PGE + i), EPI);
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);

    // the CTA's rows of phi as the B operand of phi G, [phi_hi | phi_lo]: row r is stream r / 64,
    // channel r % 64
    for (int r = threadIdx.x; r < C::NR; r += THREADS) {
        const int i = r / CW, c = r % CW;
        uint32_t hw[16], lw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            __nv_bfloat16 hv[2], lv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int j = 2 * e + u;
                const float v = (j < M && i < N) ? __ldg(phi + ((int64_t)i * d + c0 + c) * M + j) : 0.f;
                hv[u] = __float2bfloat16(v);
                lv[u] = __float2bfloat16(v - __bfloat162float(hv[u]));
            }
            hw[e] = pack_bf16x2(hv[0], hv[1]);
            lw[e] = pack_bf16x2(lv[0], lv[1]);
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            *reinterpret_cast<uint4*>(phs + sw128_off(r, ch)) =
                make_uint4(hw[4 * ch], hw[4 * ch + 1], hw[4 * ch + 2], hw[4 * ch + 3]);
            *reinterpret_cast<uint4*>(phs + sw128_off(r, ch + 4)) =
                make_uint4(lw[4 * ch], lw[4 * ch + 1], lw[4 * ch + 2], lw[4 * ch + 3]);
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tmem_slot;
    pdl_wait();                 // the token records are the previous kernel's; everything above is not

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        // Loads stage it into slot it % NS once the slot's previous stage is finished: its dX tile
        // (written by the epilogue over the dX_out rows it consumed) stored and its dphi MMAs done.
        if (lane == 0) {
            auto slot = [&](int it) { return smem_u32(sm + (it % NS) * C::STAGE); };
            auto finish = [&](int it) {
                const uint32_t ph = (uint32_t)(it / NS) & 1u;
                if (!wait(bar(B_EPID + it % NS), ph, E_EMPTY)) return false;
                tma_store_3d(&maps.dxo, slot(it) + C::XB, c0, t_lo + it * TT, 0);
                bulk_wait_read_all();
                return wait(bar(B_DPHID + it % NS), ph, E_EMPTY);
            };
            int issued = 0, finished = 0;
            bool ok = true;
            for (int it = 0; it < nst; ++it) {
                if (stop_stage >= 0 && it >= stop_stage) break;   // failure-path test hook
                if (it >= NS) {
                    if (!(ok = finish(it - NS))) break;
                    finished = it - NS + 1;
                }
                const int st = it % NS;
                const uint32_t base = slot(it);
                const uint32_t fullg = bar(B_FULLG + st), full = bar(B_FULL + st);
                const int t0 = t_lo + it * TT;
                mbar_arrive_tx(fullg, (uint32_t)C::GB);     // the record tile first: phi G needs only it
                bulk_g2s(base + 2 * C::XB + C::DXB, rec + (int64_t)(t0 / BWD_REC_TILE) * C::GB, (uint32_t)C::GB, fullg);
                mbar_arrive_tx(full, (uint32_t)(C::STAGE - C::GB));
                tma_load_3d(base, &maps.x, full, c0, t0, 0);
                tma_load_3d(base + C::XB, &maps.dy, full, c0, t0, 0);
                tma_load_2d(base + 2 * C::XB, &maps.dx, full, c0, t0);
                issued = it + 1;
            }
            for (int it = finished; ok && it < issued; ++it) {
                if (!(ok = finish(it))) break;
                finished = it + 1;
            }
            // after a failed wait: the loads of unfinished stages must have landed before the CTA exits
            for (int it = finished; it < issued; ++it) {
                drain(bar(B_FULLG + it % NS), (uint32_t)(it / NS) & 1u, E_DRAIN, false);
                drain(bar(B_FULL + it % NS), (uint32_t)(it / NS) & 1u, E_DRAIN, false);
            }
            bulk_wait_all();
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_DPHI = idesc(128, 64, 1, 1);   // A = X^T, B = [G_hi | G_lo], MN-major
            constexpr uint32_t ID_PG = idesc(64, PGN, 0, 0);     // A = G rows, B = phi rows, K-major
            // phi G over K = 96 as three products of K = 32: G_hi phi_hi, G_lo phi_hi, G_hi phi_lo
            // (byte offsets of each K16 step in the 128-byte rows of A and B)
            constexpr uint32_t AOFF[KP16] = {0, 32, 64, 96, 0, 32};
            constexpr uint32_t BOFF[KP16] = {0, 32, 0, 32, 64, 96};
            const uint32_t ph = smem_u32(phs);
            for (int it = 0; it < nst; ++it) {
                const int st = it % NS, buf = it & 1;
                if (!wait(bar(B_FULLG + st), (uint32_t)(it / NS) & 1u, E_FULL)) break;
                if (it >= NBUF && !wait(bar(B_PGE + buf), (uint32_t)((it >> 1) - 1) & 1u, E_PGEMPTY)) break;
                tc_fence_after();
                const uint32_t xs = smem_u32(sm + st * C::STAGE);
                const uint32_t gs = xs + 2 * C::XB + C::DXB;
                // phi G first (the epilogue waits for it): pair b of streams into lanes 16 b .. 16 b + 15
                // of each lane quarter
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int k = 0; k < KP16; ++k)
                        mma_bf16(tm + ((uint32_t)(16 * b) << 16) + C::PG_COL + buf * PGN, sw128_desc(gs + AOFF[k]),
                                 sw128_desc(ph + b * PGN * ROW + BOFF[k]), ID_PG, k > 0 ? 1u : 0u);
                mma_commit(bar(B_PGF + buf));
                // dphi once X has landed
                if (!wait(bar(B_FULL + st), (uint32_t)(it / NS) & 1u, E_FULL)) break;
                tc_fence_after();
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int k = 0; k < TT / 16; ++k)
                        mma_bf16(tm + C::DPHI_COL + 64 * b,
                                 sw128_desc_mn(xs + 2 * b * TT * ROW + k * 2048, TT * ROW, 1024),
                                 sw128_desc_mn(gs + k * 2048, TT * ROW, 1024), ID_DPHI,
                                 (it > 0 || k > 0) ? 1u : 0u);
                mma_commit(bar(B_DPHID + st));
            }
            // every MMA issued so far; TMEM must be idle before it is freed, and the dphi
            // partials are read after this
            mma_commit(bar(B_MMAD));
            drain(bar(B_MMAD), 0u, E_DRAIN, false);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- dX epilogue
        // thread: token row tl of the stage, stream pair hp (TMEM lanes 16 hp.. of the quarter),
        // channels [cb, cb + 32) of the slice.  dX goes over the stage's dX_out rows of the thread's
        // two streams once the warp has read them (the two lanes that share a row are in one warp);
        // the producer stores the tile.
        const int q = warp & 3, h = (warp - 2) >> 2;
        const int tl = 16 * q + (lane & 15), hp = lane >> 4, cb = 32 * h;
        const uint32_t tq = tm + ((uint32_t)(32 * q) << 16);
        bool ok = true;
        for (int it = 0; it < nst; ++it) {
            const int st = it % NS, buf = it & 1;
            if (!wait(bar(B_FULLG + st), (uint32_t)(it / NS) & 1u, E_FULL) ||
                !wait(bar(B_FULL + st), (uint32_t)(it / NS) & 1u, E_FULL) ||
                !wait(bar(B_PGF + buf), (uint32_t)(it >> 1) & 1u, E_PGFULL)) {
                ok = false;
                break;
            }
            tc_fence_after();
            unsigned char* xs = sm + st * C::STAGE;
            unsigned char* ys = xs + C::XB;
            const unsigned char* ds = xs + 2 * C::XB;
            const unsigned char* cs = ds + C::DXB + BWD_REC_TILE * 128;      // coefficient rows
            // the token's coefficients for the thread's two streams: H_pre[i], H_res[0..3][i], -beta
            float cf[2][8];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int i = (2 * hp + j) & 3;
                const uint4 a = *reinterpret_cast<const uint4*>(cs + tl * 128 + (((2 * i) ^ (tl & 7)) << 4));
                const uint4 b = *reinterpret_cast<const uint4*>(cs + tl * 128 + (((2 * i + 1) ^ (tl & 7)) << 4));
                cf[j][0] = __uint_as_float(a.x); cf[j][1] = __uint_as_float(a.y);
                cf[j][2] = __uint_as_float(a.z); cf[j][3] = __uint_as_float(a.w);
                cf[j][4] = __uint_as_float(b.x); cf[j][5] = __uint_as_float(b.y);
                cf[j][6] = __uint_as_float(b.z); cf[j][7] = __uint_as_float(b.w);
            }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t pg[2][8];
                tmem_ld_x<8>(tq + C::PG_COL + buf * PGN + cb + 8 * cc, pg[0]);        // stream 2 hp
                tmem_ld_x<8>(tq + C::PG_COL + buf * PGN + CW + cb + 8 * cc, pg[1]);   // stream 2 hp + 1
                const uint32_t roff = sw128_off(tl, 4 * h + cc);
                const uint4 dxw = *reinterpret_cast<const uint4*>(ds + roff);
                uint4 dyw[N], xw[2];
#pragma unroll
                for (int p = 0; p < N; ++p) dyw[p] = *reinterpret_cast<const uint4*>(ys + p * TT * ROW + roff);
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    xw[j] = 2 * hp + j < N ? *reinterpret_cast<const uint4*>(xs + (2 * hp + j) * TT * ROW + roff)
                                           : make_uint4(0, 0, 0, 0);
                tmem_wait8(pg[0]);
                tmem_wait8(pg[1]);
                float o[2][8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    auto word = [&](const uint4& w) { return (e >> 1) == 0 ? w.x : (e >> 1) == 1 ? w.y : (e >> 1) == 2 ? w.z : w.w; };
                    auto unpack = [&](const uint4& w) { return (e & 1) ? bf_hi(word(w)) : bf_lo(word(w)); };
                    const float dxv = unpack(dxw);
                    float dyv[N];
#pragma unroll
                    for (int p = 0; p < N; ++p) dyv[p] = unpack(dyw[p]);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        float v = fmaf(cf[j][0], dxv, __uint_as_float(pg[j][e]));
                        v = fmaf(cf[j][5], unpack(xw[j]), v);
#pragma unroll
                        for (int p = 0; p < N; ++p) v = fmaf(cf[j][1 + p], dyv[p], v);
                        o[j][e] = v;
                    }
                }
                __syncwarp();     // every lane of the warp has read this chunk's dX_out rows
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int i = 2 * hp + j;
                    if (i >= N) continue;
                    *reinterpret_cast<uint4*>(ys + i * TT * ROW + roff) =
                        make_uint4(pack_f32x2(o[j][0], o[j][1]), pack_f32x2(o[j][2], o[j][3]),
                                   pack_f32x2(o[j][4], o[j][5]), pack_f32x2(o[j][6], o[j][7]));
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the tile is read by a TMA store
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_PGE + buf));
                mbar_arrive(bar(B_EPID + st));
            }
        }
        // dphi partials of the group: warps h = b read block b (TMEM lane = row k of the block)
        if (ok && h < NB && !wait(bar(B_MMAD), 0u, E_DRAIN)) ok = false;
        if (ok && h < NB) {
            const int i = 2 * h + (q >> 1), c = 32 * (q & 1) + lane;
            if (i < N) {
                float* dst = part + ((int64_t)g * K + (int64_t)i * d + c0 + c) * M;
                if (nst > 0) {
#pragma unroll
                    for (int j0 = 0; j0 < M; j0 += 16) {      // hi columns j, lo columns 32 + j
                        uint32_t vh[16], vl[16];
                        tmem_ld_x<16>(tq + C::DPHI_COL + 64 * h + j0, vh);
                        tmem_ld_x<16>(tq + C::DPHI_COL + 64 * h + 32 + j0, vl);
                        tmem_wait16(vh);
                        tmem_wait16(vl);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (j0 + j < M) dst[j0 + j] = __uint_as_float(vh[j]) + __uint_as_float(vl[j]);
                    }
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

// failure-path test hook (mhc_debug_backward_stop_after): stages per CTA after which the
// producer stops loading (< 0: never), and the wait limit
std::atomic<int> g_stop_stage{-1};
std::atomic<unsigned long long> g_wait_ns{kWaitNs};

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
    {   // dX (stores): the view of X
        const cuuint64_t dims[3] = {(cuuint64_t)a.d, (cuuint64_t)a.T, (cuuint64_t)N};
        const cuuint64_t str[2] = {(cuuint64_t)N * a.d * 2, (cuuint64_t)a.d * 2};
        const cuuint32_t box[3] = {CW, TT, N};
        r = enc(&maps.dxo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.dX, dims, str, box, e1,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    const int slices = a.d / CW;
    const unsigned grid = (unsigned)(slices * groups);
    return launch_pdl(bwd_tc_kernel<N>, dim3(grid), dim3(THREADS), (size_t)Cfg<N>::SMEM, a.stream, maps, a.phi,
                      static_cast<const unsigned char*>(rec), (int)a.T, a.d, (int)tpg,
                      static_cast<__nv_bfloat16*>(a.dX), part, g_stop_stage.load(), g_wait_ns.load());
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

void bwd_tc_set_stop(int stop_stage, unsigned long long wait_ns) {
    bwdtc::g_stop_stage.store(stop_stage);
    bwdtc::g_wait_ns.store(wait_ns);
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
