// pre_wide.cu -- the mHC pre stage on B200 tensor cores for the shapes whose phi does not
// fit the shared memory of one 16-CTA cluster: n = 5..8 streams (phi at n = 8, d = 4096 is
// 10 MB), or n <= 4 with a large d.
//
// What it computes is the pre stage of "DeepSeek-V4/mhc" (equations rmsnorm, a/b/c-tilde,
// gate, sinkhorn-init, sinkhorn) and the read map H_pre x_l of the slavadubrov.com Eq. 3
// (or, with hc set, the HC maps b + alpha tanh(h)); see include/mhc.h.  Three launches:
//
//   1. pack: phi (fp32, [n d, m]) -> the shared-memory image of the MMA's B operand, one
//      64-channel atom at a time: rows [0, m) phi_hi = bf16(phi), rows [MH, MH + m)
//      phi_lo = bf16(phi - phi_hi) (16 significant bits, above the TF32 the mixed-
//      precision table asks for), K-major with the 128-byte swizzle.  It is written into
//      the x_in buffer, which holds nothing else until launch 3 writes x_in.
//   2. projection: clusters of C = 4 CTAs split K = n d; a cluster takes 256-token tiles
//      (4-CTA clusters fill the GPU in one wave of tiles at the n = 8 workload).
//      A stage holds one 64-channel atom: the tile's X (a 32 KB TMA box) and that atom of
//      packed phi (a bulk copy, served from L2); four stages keep about 200 KB in flight per
//      SM.  Two warps issue tcgen05.mma (M = 128 tokens, N = 2 MH, K = 16), one per half of
//      the tile, into TMEM; four warps add the tokens' squares.  Each CTA writes its partial
//      projection and sum of squares of every token to a scratch block in the x_in buffer;
//      the owner CTA of a token (64 tokens each) adds the 4 partials in a fixed order into
//      shared memory with coalesced loads, applies 1/r and forms H.  For a CTA's last tile
//      every warp takes part (the stage ring is idle by then): four threads per token, the
//      Sinkhorn rows split between them.
//   3. read map: x_in = sum_i H_pre[i] X[i, :], streaming X from HBM a second time.
//
// X crosses HBM twice here; streaming phi instead against tiles small enough to re-read
// X from L2 would cost more than one read of X in phi traffic.  Every wait on an mbarrier
// is bounded in time (status word: mhc_device_status).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.cuh"
#include "tc_ptx.cuh"

namespace mhc {

// Status of this path's bounded waits since the last read (0 = fine).
__device__ unsigned int g_pre_wide_status;

namespace wide {

constexpr int C = 4;               // CTAs per cluster (K split)
constexpr int TT = 256;            // tokens per tile
constexpr int HALF = 128;          // MMA M
constexpr int TPO = TT / C;        // tokens owned per CTA and tile
constexpr int NS = 2;              // partial-arrival barrier ring
constexpr int MAXST = 6;
constexpr int NWARPS = 8;          // 0 TMA, 1-2 MMA, 3 owner, 4-7 squares + epilogue
constexpr int THREADS = NWARPS * 32;
constexpr int TMEM_COLS = 512;
constexpr int X_STAGE = TT * 128;  // one atom of a 256-token tile
constexpr int SW = 1;              // atoms per stage (one 32 KB box of X, one copy of phi; measured
                                   // slightly faster than two atoms per stage)
constexpr unsigned long long kWaitNs = 1000000000ull;

static_assert(TPO % 32 == 0, "the owner warp takes TPO / 32 tokens per lane");
static_assert(THREADS == 4 * TPO && TPO % NWARPS == 0, "the last tile's maps: four threads per owned token");

template <int N>
struct Cfg {
    static constexpr int M = N * N + 2 * N;
    static constexpr int MH = (M + 15) / 16 * 16;          // hi rows, padded to 16
    static constexpr int NB = 2 * MH;                      // MMA N: [hi | lo]
    static constexpr int PHI_ATOM = NB / 8 * 1024;         // bytes of one packed atom
    static constexpr int W = ((MH > M + 1 ? MH : M + 1) + 3) / 4 * 4;   // floats per partial record
    static constexpr int STAGE = SW * (X_STAGE + PHI_ATOM);
    static constexpr int HSW = W | 1;                      // owner buffer row stride (odd: no bank conflicts)
    static constexpr int HS = 32 * HSW * 4;                // owner: summed records of 32 tokens
    static constexpr int NACCB = TMEM_COLS / (2 * NB) >= 2 ? 2 : 1;     // accumulator buffers
    static_assert(NB <= 256 && NB % 16 == 0, "MMA N for M = 128");
    static_assert(2 * NB <= TMEM_COLS, "both halves fit TMEM");
};

__host__ __device__ constexpr uint32_t idesc_m128(int nb) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(nb >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

enum : int {
    B_FULL = 0, B_EMPTY = MAXST, B_ACCF = 2 * MAXST, B_ACCE = B_ACCF + 2, B_EPI = B_ACCE + 2,
    B_PFULL = B_EPI + 1, B_PEMPTY = B_PFULL + NS, B_DRAIN = B_PEMPTY + NS, B_COUNT = B_DRAIN + 2
};
enum : unsigned {
    E_EMPTY = 1u, E_FULL = 2u, E_ACCE = 4u, E_ACCF = 8u, E_EPI = 16u, E_PEMPTY = 32u, E_PFULL = 64u,
    E_DRAIN = 128u
};

using namespace ptx;

struct Waiter {
    volatile int* abort_flag;
    unsigned long long limit_ns;
    template <bool CLUSTER = false>
    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity, unsigned code,
                                               bool honour_abort = true) const {
        auto try_once = [&]() { return CLUSTER ? mbar_try_cluster(bar, parity) : mbar_try(bar, parity); };
        if (try_once()) return true;
        const uint64_t t0 = gtimer();
        while (true) {
            if (try_once()) return true;
            if (honour_abort && *abort_flag) return false;
            if (gtimer() - t0 > limit_ns) {
                atomicOr(&g_pre_wide_status, code);
                *abort_flag = 1;
                return false;
            }
        }
    }
};

struct WMaps {
    CUtensorMap box[SW];           // box[j]: j + 1 atoms of a 256-token tile
};

__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_wait_regs16(uint32_t* r) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                   "+r"(r[13]), "+r"(r[14]), "+r"(r[15]) :: "memory");
}

// ---------------------------------------------------------------- 1. pack
// One thread per (atom, 8-value chunk, B row): 16 bytes of the atom's swizzled image.
template <int N>
__global__ void __launch_bounds__(256)
wide_pack_kernel(const float* __restrict__ phi, int ka_total, uint8_t* __restrict__ packed)
{
    using Cf = Cfg<N>;
    constexpr int M = Cf::M, MH = Cf::MH, NB = Cf::NB;
    const int64_t total = (int64_t)ka_total * 8 * NB;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int j = (int)(e % NB);
        const int64_t ac = e / NB;
        const int c8 = (int)(ac % 8);
        const int64_t a = ac / 8;
        const bool lo = j >= MH;
        const int col = lo ? j - MH : j;
        float v[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            float out = 0.f;
            if (col < M) {
                const float p = __ldg(phi + (a * 64 + c8 * 8 + x) * M + col);
                const float hi = __bfloat162float(__float2bfloat16_rn(p));
                out = lo ? p - hi : hi;
            }
            v[x] = out;
        }
        *reinterpret_cast<uint4*>(packed + a * Cf::PHI_ATOM + sw128_off(j, c8)) = Vec16<__nv_bfloat16>::pack(v);
    }
}

// ---------------------------------------------------------------- 2. projection
// The maps of one token from its summed projection hv (length m, not yet divided by r), four
// lanes per token ("DeepSeek-V4/mhc", equations a/b/c-tilde, gate, sinkhorn-init, sinkhorn;
// the HC maps b + alpha tanh(h / r) when hc): lane gl of the group owns rows 2 gl and 2 gl + 1
// (those below N).  In each Sinkhorn round a column sum adds the lanes' two-row sums by xor
// shuffles within the group (every lane gets the same sum); row sums are the lane's own.  All
// four lanes run the shuffles; only `valid` tokens are written.
template <int N>
__device__ __forceinline__ void owner_maps4(const float* hv, float inv_r, int gl, const float* b_pre,
                                            const float* b_post, const float* b_res, float a_pre, float a_post,
                                            float a_res, int t_max, bool hc, bool valid, float* Hrow, float* hrow) {
    static_assert(N <= 8, "two rows per lane, four lanes per token");
    float Mx[2][N];
    bool own[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int i = 2 * gl + r;
        own[r] = i < N;
#pragma unroll
        for (int j = 0; j < N; ++j)
            Mx[r][j] = (own[r] && !hc) ? expf(a_res * (hv[N + i * N + j] * inv_r) + b_res[i * N + j]) : 0.f;
    }
    if (!hc) {
        // each step over all N columns at once, so the shuffles and divisions of different
        // columns overlap
        for (int it = 0; it < t_max; ++it) {
            float cs[N];
#pragma unroll
            for (int j = 0; j < N; ++j) cs[j] = Mx[0][j] + Mx[1][j];
#pragma unroll
            for (int j = 0; j < N; ++j) cs[j] += __shfl_xor_sync(0xffffffffu, cs[j], 1);
#pragma unroll
            for (int j = 0; j < N; ++j) cs[j] += __shfl_xor_sync(0xffffffffu, cs[j], 2);
#pragma unroll
            for (int j = 0; j < N; ++j) cs[j] = __fdividef(1.0f, cs[j]);
#pragma unroll
            for (int j = 0; j < N; ++j) {
                Mx[0][j] *= cs[j];
                Mx[1][j] *= cs[j];
            }
            float rs[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < N; ++j) s += Mx[r][j];
                rs[r] = own[r] ? __fdividef(1.0f, s) : 0.f;
            }
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int j = 0; j < N; ++j) Mx[r][j] *= rs[r];
        }
    }
    if (!valid) return;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (!own[r]) continue;
        const int i = 2 * gl + r;
        const float zp = hv[i] * inv_r, zq = hv[N + N * N + i] * inv_r;
        Hrow[i] = hc ? b_pre[i] + a_pre * tanhf(zp) : sigmoid_f32(a_pre * zp + b_pre[i]);
        Hrow[N + N * N + i] = hc ? b_post[i] + a_post * tanhf(zq) : 2.0f * sigmoid_f32(a_post * zq + b_post[i]);
#pragma unroll
        for (int j = 0; j < N; ++j)
            Hrow[N + i * N + j] = hc ? b_res[i * N + j] + a_res * tanhf(hv[N + i * N + j] * inv_r) : Mx[r][j];
        if (hrow != nullptr) {
            hrow[i] = zp;
            hrow[N + N * N + i] = zq;
#pragma unroll
            for (int j = 0; j < N; ++j) hrow[N + i * N + j] = hv[N + i * N + j] * inv_r;
        }
    }
}

// The C partial records of tokens [u0, u0 + nu) of a tile added in source order, the lanes along
// the record (coalesced loads), into rows u0.. of hs (row stride HSW).
template <int W, int HSW>
__device__ __forceinline__ void sum_records(const float* __restrict__ blk, int rank, int u0, int nu, int lane,
                                            float* hs, int hs_row0) {
    constexpr int QW = (W + 31) / 32;
#pragma unroll 1
    for (int v0 = 0; v0 < nu; v0 += 4) {
        float acc[4][QW];
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
            const float* rec = blk + ((int64_t)(rank * TPO + u0 + v0 + uu) * C) * W;
#pragma unroll
            for (int q = 0; q < QW; ++q) {
                const int j = lane + 32 * q;
                float v = 0.f;
                if (j < W && v0 + uu < nu) {
#pragma unroll
                    for (int src = 0; src < C; ++src) v += __ldcg(rec + src * W + j);
                }
                acc[uu][q] = v;
            }
        }
#pragma unroll
        for (int uu = 0; uu < 4; ++uu)
#pragma unroll
            for (int q = 0; q < QW; ++q)
                if (lane + 32 * q < W && v0 + uu < nu) hs[(hs_row0 + v0 + uu) * HSW + lane + 32 * q] = acc[uu][q];
    }
}

template <int N>
__global__ void __launch_bounds__(THREADS, 1)
wide_proj_kernel(const __grid_constant__ WMaps maps, const uint8_t* __restrict__ packed,
                 float* __restrict__ scratch, const float* __restrict__ b_pre,
                 const float* __restrict__ b_post, const float* __restrict__ b_res, float a_pre,
                 float a_post, float a_res, int T, int d, float eps, int t_max,
                 float* __restrict__ H, float* __restrict__ h_out, int ka_total, int nstage,
                 int hc, unsigned long long wait_ns)
{
    using Cf = Cfg<N>;
    constexpr int M = Cf::M, MH = Cf::MH, NB = Cf::NB, W = Cf::W, NACCB = Cf::NACCB, HSW = Cf::HSW;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* sb = smem_raw + (base - raw);
    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int a_lo = (int)(((int64_t)rank * ka_total) / C);
    const int ka = (int)((((int64_t)rank + 1) * ka_total) / C) - a_lo;

    const uint32_t o_bar = (uint32_t)nstage * Cf::STAGE;
    const uint32_t o_misc = o_bar + B_COUNT * 8u;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sb + o_misc);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sb + o_misc + 4);
    float* hs = reinterpret_cast<float*>(sb + o_misc + 16);
    auto bar = [&](int i) -> uint32_t { return base + o_bar + 8u * (uint32_t)i; };
    const Waiter wait{abort_flag, wait_ns};
    const Waiter drain{abort_flag, wait_ns > kWaitNs ? wait_ns : kWaitNs};

    const int num_tiles = (T + TT - 1) / TT;
    const int cid = (int)cluster_idx(), ncl = (int)cluster_count();
    const int my_tiles = cid < num_tiles ? (num_tiles - cid + ncl - 1) / ncl : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; ++s) {
            mbar_init(bar(B_FULL + s), 1);
            mbar_init(bar(B_EMPTY + s), 2 + 4);          // two issuers' commits + 4 squares warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_ACCF + b), 2);
            mbar_init(bar(B_ACCE + b), 4);
        }
        mbar_init(bar(B_EPI), 4);                          // the epilogue warps wrote their partials
        for (int sl = 0; sl < NS; ++sl) {
            mbar_init(bar(B_PFULL + sl), C);              // one arrive per source CTA
            mbar_init(bar(B_PEMPTY + sl), C);             // one arrive per owner CTA
        }
        for (int i = 0; i < 2; ++i) mbar_init(bar(B_DRAIN + i), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), (uint32_t)TMEM_COLS);
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();                 // packed phi and the scratch belong to the packing launch

    if (warp == 0) {
        // producer: stage g = (tile g / spt, atoms from al = (g % spt) * SW): one X box of
        // na atoms and one copy of their packed phi
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.box[SW - 1]) : "memory");
            const int spt = (ka + SW - 1) / SW;
            const int total = my_tiles * spt;
            int g = 0;
            for (; g < total; ++g) {
                const int k = g / spt, al = (g - k * spt) * SW;
                const int na = ka - al < SW ? ka - al : SW;
                const int s = g % nstage, u = g / nstage;
                if (!wait(bar(B_EMPTY + s), (u & 1) ^ 1, E_EMPTY)) break;
                const uint32_t st = base + (uint32_t)s * Cf::STAGE;
                mbar_arrive_tx(bar(B_FULL + s), (uint32_t)(na * (X_STAGE + Cf::PHI_ATOM)));
                tma_load_3d(st, &maps.box[na - 1], bar(B_FULL + s), 0, (cid + k * ncl) * TT, a_lo + al);
                bulk_g2s(st + SW * X_STAGE, packed + (int64_t)(a_lo + al) * Cf::PHI_ATOM,
                         (uint32_t)(na * Cf::PHI_ATOM), bar(B_FULL + s));
            }
            for (int j = g - 1; j >= 0 && j >= g - nstage; --j)
                drain(bar(B_FULL + j % nstage), (j / nstage) & 1, E_DRAIN, false);
        }
        __syncwarp();
    } else if (warp == 1 || warp == 2) {
        // MMA issuer for half h of every tile
        const int h = warp - 1;
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_m128(NB);
            int g = 0, issued = 0;
            bool stop = false;
            for (int k = 0; k < my_tiles && !stop; ++k) {
                const int b = k % NACCB, ub = k / NACCB;
                if (!wait(bar(B_ACCE + b), (ub & 1) ^ 1, E_ACCE)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)((b * 2 + h) * NB);
                for (int al = 0; al < ka; al += SW, ++g) {
                    const int na = ka - al < SW ? ka - al : SW;
                    const int s = g % nstage, u = g / nstage;
                    if (!wait(bar(B_FULL + s), u & 1, E_FULL)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t st = base + (uint32_t)s * Cf::STAGE;
                    for (int j = 0; j < na; ++j) {
                        const uint64_t ad = sw128_desc(st + (uint32_t)(j * X_STAGE + h * (HALF * 128)));
                        const uint64_t bd = sw128_desc(st + (uint32_t)(SW * X_STAGE + j * Cf::PHI_ATOM));
                        mma_bf16(d_tmem, ad, bd, IDESC, (al > 0 || j > 0) ? 1u : 0u);
                        mma_bf16(d_tmem, ad + 2, bd + 2, IDESC, 1);
                        mma_bf16(d_tmem, ad + 4, bd + 4, IDESC, 1);
                        mma_bf16(d_tmem, ad + 6, bd + 6, IDESC, 1);
                    }
                    issued = 1;
                    mma_commit(bar(B_EMPTY + s));
                }
                if (stop) break;
                mma_commit(bar(B_ACCF + b));
            }
            if (issued) {
                mma_commit(bar(B_DRAIN + h));
                drain(bar(B_DRAIN + h), 0, E_DRAIN, false);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // squares (thread = tokens 32q + lane of both halves), then the epilogue: TMEM lane
        // 32q + lane holds the same token of each half
        const int q = warp - 4;
        const int r0 = 32 * q + lane, r1 = HALF + r0;
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        int g = 0;
        for (int k = 0; k < my_tiles; ++k) {
            float2 s0[4], s1[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) s0[x] = s1[x] = make_float2(0.f, 0.f);
            bool ok = true;
            for (int al = 0; al < ka; al += SW, ++g) {
                const int na = ka - al < SW ? ka - al : SW;
                const int s = g % nstage, u = g / nstage;
                if (!wait(bar(B_FULL + s), u & 1, E_FULL)) { ok = false; break; }
                for (int j = 0; j < na; ++j) {
                    const uint8_t* st = sb + (uint32_t)s * Cf::STAGE + (uint32_t)j * X_STAGE;
                    uint4 w0[8], w1[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        w0[c] = *reinterpret_cast<const uint4*>(st + r0 * 128 + ((c ^ (r0 & 7)) << 4));
                        w1[c] = *reinterpret_cast<const uint4*>(st + r1 * 128 + ((c ^ (r1 & 7)) << 4));
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t a0[4] = {w0[c].x, w0[c].y, w0[c].z, w0[c].w};
                        const uint32_t a1[4] = {w1[c].x, w1[c].y, w1[c].z, w1[c].w};
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const float2 f0 = bf16x2_to_f32x2(a0[x]), f1 = bf16x2_to_f32x2(a1[x]);
                            s0[x] = __ffma2_rn(f0, f0, s0[x]);
                            s1[x] = __ffma2_rn(f1, f1, s1[x]);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_EMPTY + s));
            }
            if (!ok) break;
            const float ss[2] = {((s0[0].x + s0[0].y) + (s0[1].x + s0[1].y)) + ((s0[2].x + s0[2].y) + (s0[3].x + s0[3].y)),
                                 ((s1[0].x + s1[0].y) + (s1[1].x + s1[1].y)) + ((s1[2].x + s1[2].y) + (s1[3].x + s1[3].y))};
            const int b = k % NACCB, ub = k / NACCB;
            if (!wait(bar(B_ACCF + b), ub & 1, E_ACCF)) break;
            tc_fence_after();
            // record [h partial (hi + lo) | sum of squares | pad] of token t of tile k, this CTA
            const int tile = cid + k * ncl;
            float* blk = scratch + (int64_t)tile * TT * C * W;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = h * HALF + r0;
                float* rec = blk + ((int64_t)t * C + rank) * W;
#pragma unroll
                for (int c = 0; c < MH / 16; ++c) {
                    uint32_t rh[16], rl[16];
                    tmem_ld16_nowait(tq + (uint32_t)((b * 2 + h) * NB + c * 16), rh);
                    tmem_ld16_nowait(tq + (uint32_t)((b * 2 + h) * NB + MH + c * 16), rl);
                    tmem_wait_regs16(rh);
                    tmem_wait_regs16(rl);
#pragma unroll
                    for (int x4 = 0; x4 < 4; ++x4) {
                        float4 v;
                        v.x = __uint_as_float(rh[4 * x4 + 0]) + __uint_as_float(rl[4 * x4 + 0]);
                        v.y = __uint_as_float(rh[4 * x4 + 1]) + __uint_as_float(rl[4 * x4 + 1]);
                        v.z = __uint_as_float(rh[4 * x4 + 2]) + __uint_as_float(rl[4 * x4 + 2]);
                        v.w = __uint_as_float(rh[4 * x4 + 3]) + __uint_as_float(rl[4 * x4 + 3]);
                        *reinterpret_cast<float4*>(rec + c * 16 + 4 * x4) = v;
                    }
                }
                rec[M] = ss[h];
            }
            tc_fence_before();
            __threadfence();                  // the records are visible GPU-wide before the signal
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_ACCE + b));
                mbar_arrive(bar(B_EPI));
            }
            if (q == 0) {
                // tell the C owners that this CTA's records of tile k are written, once every
                // owner has consumed this CTA's signal of tile k - NS
                if (!wait(bar(B_EPI), k & 1, E_EPI)) break;
                const int sl = k % NS, us = k / NS;
                if (lane < C && wait(bar(B_PEMPTY + sl), (us & 1) ^ 1, E_PEMPTY)) {
                    asm volatile("fence.acq_rel.cluster;" ::: "memory");
                    mbar_arrive_remote(mapa(bar(B_PFULL + sl), (uint32_t)lane));
                }
                __syncwarp();
            }
        }
    } else if (warp == 3) {
        // owner of every tile but the last (whose owner phase all warps share, below): tokens
        // rank * TPO .. rank * TPO + TPO - 1, 32 at a time, record sums into hs, then the maps
        // one lane per token
        for (int k = 0; k + 1 < my_tiles; ++k) {
            const int sl = k % NS, us = k / NS;
            if (!wait.template operator()<true>(bar(B_PFULL + sl), us & 1, E_PFULL)) break;
            const int tile = cid + k * ncl;
            const float* blk = scratch + (int64_t)tile * TT * C * W;
#pragma unroll 1
            for (int half = 0; half < TPO / 32; ++half) {
                sum_records<W, HSW>(blk, (int)rank, half * 32, 32, lane, hs, 0);
                if (half == TPO / 32 - 1) {   // every record of this tile has been read
                    __syncwarp();
                    if (lane < C) mbar_arrive_remote(mapa(bar(B_PEMPTY + sl), (uint32_t)lane));
                }
                __syncwarp();                 // hs is complete before the maps read it
                const int64_t tok = (int64_t)tile * TT + (int)rank * TPO + half * 32 + lane;
                const float* hv = hs + lane * HSW;
                const float inv_r = 1.0f / sqrtf(hv[M] / (float)(N * d) + eps);
                if (tok < T) {
                    if (h_out != nullptr) {
#pragma unroll
                        for (int j = 0; j < M; ++j) h_out[tok * M + j] = hv[j] * inv_r;
                    }
                    float out[M];
                    if (hc) token_maps_hc<N>(hv, inv_r, b_pre, b_post, b_res, a_pre, a_post, a_res, out);
                    else token_maps<N>(hv, inv_r, b_pre, b_post, b_res, a_pre, a_post, a_res, t_max, out);
#pragma unroll
                    for (int j = 0; j < M; ++j) H[tok * M + j] = out[j];
                }
                __syncwarp();                 // the maps have read hs before the next half fills it
            }
        }
    }

    // ---- the last tile's owner phase, all warps: the stage ring is idle once every role has
    // left its loop (loads drained, MMAs complete), so it holds the 64 tokens' summed records;
    // each warp sums 8 tokens' records, then four threads form each token's maps
    if (my_tiles > 0) {
        const int k = my_tiles - 1, sl = k % NS, us = k / NS;
        volatile int* go = reinterpret_cast<volatile int*>(sb + o_misc + 8);
        if (warp == 3) {
            const bool ok = !*abort_flag && wait.template operator()<true>(bar(B_PFULL + sl), us & 1, E_PFULL);
            if (lane == 0) *go = ok ? 1 : 0;
        }
        __syncthreads();
        if (*go) {
            const int tile = cid + k * ncl;
            float* hsl = reinterpret_cast<float*>(sb);
            sum_records<W, HSW>(scratch + (int64_t)tile * TT * C * W, (int)rank, warp * (TPO / NWARPS),
                                TPO / NWARPS, lane, hsl, warp * (TPO / NWARPS));
            __syncthreads();
            if (warp == 3 && lane < C) mbar_arrive_remote(mapa(bar(B_PEMPTY + sl), (uint32_t)lane));
            const int u = threadIdx.x >> 2, gl = threadIdx.x & 3;
            const int64_t tok = (int64_t)tile * TT + (int)rank * TPO + u;
            const float* hv = hsl + u * HSW;
            const float inv_r = 1.0f / sqrtf(hv[M] / (float)(N * d) + eps);
            owner_maps4<N>(hv, inv_r, gl, b_pre, b_post, b_res, a_pre, a_post, a_res, t_max, hc != 0, tok < T,
                           H + tok * M, h_out != nullptr ? h_out + tok * M : nullptr);
        }
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)TMEM_COLS);
    }
}

// ---------------------------------------------------------------- 3. read map
// One warp task = (token, 32 chunks of 8 channels); x_in = sum_i H_pre[i] X_i.
template <int N>
__global__ void __launch_bounds__(256)
wide_xin_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ H, int64_t Tn, int d,
                __nv_bfloat16* __restrict__ x_in)
{
    constexpr int M = N * N + 2 * N;
    const int chunks = d / 8;
    const int per_tok = (chunks + 31) >> 5;
    const int64_t ntasks = Tn * per_tok;
    const int lane = threadIdx.x & 31;
    pdl_wait();                 // H is the projection launch's
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t task = (((int64_t)blockIdx.x * blockDim.x) + threadIdx.x) >> 5; task < ntasks; task += nwarps) {
        const int64_t t = task / per_tok;
        const int c = (int)(task - t * per_tok) * 32 + lane;
        float hp[N];
#pragma unroll
        for (int i = 0; i < N; ++i) hp[i] = __ldg(H + t * M + i);
        if (c < chunks) {
            uint4 xv[N];
#pragma unroll
            for (int i = 0; i < N; ++i) xv[i] = ld_stream_v4(X + (t * N + i) * (int64_t)d + (int64_t)c * 8);
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
            for (int i = 0; i < N; ++i) {
                float f[8];
                Vec16<__nv_bfloat16>::unpack(xv[i], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(hp[i], f[e], acc[e]);
            }
            st_v4(x_in + t * (int64_t)d + (int64_t)c * 8, Vec16<__nv_bfloat16>::pack(acc));
        }
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    bool ok = false;
    int nstage = 0, smem = 0, max_clusters = 0;
};

template <int N>
int smem_bytes(int nstage) { return nstage * Cfg<N>::STAGE + B_COUNT * 8 + 16 + Cfg<N>::HS + 1024; }

template <int N>
Plan make_plan() {
    Plan p;
    DeviceInfo di;
    if (device_info(&di) != cudaSuccess || di.cc_major != 10 || di.cc_minor != 0) return p;
    int ns = MAXST;
    while (ns >= 2 && smem_bytes<N>(ns) > di.max_smem_optin) --ns;
    if (ns < 2) return p;
    auto kern = wide_proj_kernel<N>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, di.max_smem_optin) != cudaSuccess) {
        cudaGetLastError();
        return p;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C * 8);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem_bytes<N>(ns);
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess || nc < 1) {
        cudaGetLastError();
        return p;
    }
    p.ok = true;
    p.nstage = ns;
    p.smem = smem_bytes<N>(ns);
    p.max_clusters = nc;
    return p;
}

Plan get_plan(int n) {
    static std::mutex mu;
    static Plan cache[64][9];
    static bool have[64][9] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || n < 1 || n > 8) {
        cudaGetLastError();
        return Plan{};
    }
    std::lock_guard<std::mutex> lk(mu);
    if (!have[dev][n]) {
        Plan p;
        switch (n) {
            case 1: p = make_plan<1>(); break;
            case 2: p = make_plan<2>(); break;
            case 3: p = make_plan<3>(); break;
            case 4: p = make_plan<4>(); break;
            case 5: p = make_plan<5>(); break;
            case 6: p = make_plan<6>(); break;
            case 7: p = make_plan<7>(); break;
            case 8: p = make_plan<8>(); break;
        }
        cache[dev][n] = p;
        have[dev][n] = true;
    }
    return cache[dev][n];
}

// Bytes of the x_in buffer this path uses as scratch: the packed phi, then the partial records.
template <int N>
int64_t scratch_bytes(int64_t T, int d) {
    using Cf = Cfg<N>;
    const int64_t packed = (int64_t)(N * d / 64) * Cf::PHI_ATOM;
    const int64_t part = ((T + TT - 1) / TT) * TT * C * Cf::W * 4;
    return (packed + 255) / 256 * 256 + part;
}

int64_t scratch_bytes_n(int n, int64_t T, int d) {
    switch (n) {
        case 1: return scratch_bytes<1>(T, d);
        case 2: return scratch_bytes<2>(T, d);
        case 3: return scratch_bytes<3>(T, d);
        case 4: return scratch_bytes<4>(T, d);
        case 5: return scratch_bytes<5>(T, d);
        case 6: return scratch_bytes<6>(T, d);
        case 7: return scratch_bytes<7>(T, d);
        case 8: return scratch_bytes<8>(T, d);
    }
    return -1;
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

unsigned long long g_wait_ns = kWaitNs;

template <int N>
cudaError_t launch_n(const PreArgs& a, const Plan& p) {
    using Cf = Cfg<N>;
    const int ka_total = N * a.d / 64;
    uint8_t* packed = static_cast<uint8_t*>(a.x_in);
    const int64_t packed_bytes = ((int64_t)ka_total * Cf::PHI_ATOM + 255) / 256 * 256;
    float* scratch = reinterpret_cast<float*>(packed + packed_bytes);
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    {
        const int64_t work = (int64_t)ka_total * 8 * Cf::NB;
        int64_t blocks = (work + 255) / 256;
        if (blocks > (int64_t)di.sm_count * 8) blocks = (int64_t)di.sm_count * 8;
        wide_pack_kernel<N><<<(unsigned)blocks, 256, 0, a.stream>>>(a.phi, ka_total, packed);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        // X viewed as 3-D: (element within a 64-channel atom, token, atom); box j: (64, 256,
        // j + 1), stored atom-major
        WMaps maps;
        const cuuint64_t dims[3] = {64, (cuuint64_t)a.T, (cuuint64_t)ka_total};
        const cuuint64_t strides[2] = {(cuuint64_t)N * a.d * 2, 128};
        const cuuint32_t estr[3] = {1, 1, 1};
        auto enc = encode_fn();
        if (!enc) return cudaErrorNotSupported;
        for (int j = 0; j < SW; ++j) {
            const cuuint32_t box[3] = {64, (cuuint32_t)TT, (cuuint32_t)(j + 1)};
            if (enc(&maps.box[j], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.X), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        const int num_tiles = (int)((a.T + TT - 1) / TT);
        const int ncl = num_tiles < p.max_clusters ? num_tiles : p.max_clusters;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(ncl * C));
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = (size_t)p.smem;
        cfg.stream = a.stream;
        cudaLaunchAttribute at[2];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = C;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        // the set-up (barriers, TMEM) overlaps the packing launch's tail; pdl_wait precedes every
        // access to the packed phi and the scratch
        at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, wide_proj_kernel<N>, maps, static_cast<const uint8_t*>(packed), scratch,
                               a.b_pre, a.b_post, a.b_res, a.a_pre, a.a_post, a.a_res, (int)a.T, a.d, a.eps,
                               a.t_max, a.H, a.h_out, ka_total, p.nstage, a.hc ? 1 : 0, g_wait_ns);
        if (e != cudaSuccess) return e;
    }
    {
        const int64_t per_tok = (a.d / 8 + 31) / 32;
        int64_t blocks = (a.T * per_tok * 32 + 255) / 256;
        if (blocks > (int64_t)di.sm_count * 8) blocks = (int64_t)di.sm_count * 8;
        e = launch_pdl(wide_xin_kernel<N>, dim3((unsigned)blocks), dim3(256), 0, a.stream,
                       static_cast<const __nv_bfloat16*>(a.X), static_cast<const float*>(a.H), a.T, a.d,
                       static_cast<__nv_bfloat16*>(a.x_in));
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace wide

bool pre_wide_shape_ok(int64_t T, int n, int d, DType dt) {
    if (dt != BF16 || n < 1 || n > 8 || d % 64 != 0 || (int64_t)n * d < 64 * wide::C || T < 1 ||
        T >= ((int64_t)1 << 31) - wide::TT)
        return false;
    return wide::scratch_bytes_n(n, T, d) <= T * (int64_t)d * 2;     // fits the x_in buffer
}

bool pre_wide_device_ok(int n) { return wide::get_plan(n).ok; }

cudaError_t launch_pre_wide(const PreArgs& a) {
    const wide::Plan p = wide::get_plan(a.n);
    if (!p.ok) return cudaErrorNotSupported;
    switch (a.n) {
        case 1: return wide::launch_n<1>(a, p);
        case 2: return wide::launch_n<2>(a, p);
        case 3: return wide::launch_n<3>(a, p);
        case 4: return wide::launch_n<4>(a, p);
        case 5: return wide::launch_n<5>(a, p);
        case 6: return wide::launch_n<6>(a, p);
        case 7: return wide::launch_n<7>(a, p);
        case 8: return wide::launch_n<8>(a, p);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t pre_wide_status(unsigned* out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_pre_wide_status, sizeof(unsigned));
    if (e != cudaSuccess) return e;
    if (clear && *out) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_pre_wide_status, &zero, sizeof(unsigned));
    }
    return e;
}

}  // namespace mhc
