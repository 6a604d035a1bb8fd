// pre_cluster_tc.cu -- the mHC pre stage on B200 tensor cores, one HBM read of X.
//
// What it computes is the pre stage of "DeepSeek-V4/mhc" (equations rmsnorm, a/b/c-tilde,
// gate, sinkhorn-init, sinkhorn) and the read map H_pre x_l of the slavadubrov.com Eq. 3;
// see include/mhc.h.  How, on sm_100a:
//
//   * A cluster of S = 16 CTAs splits the channel axis: CTA c owns channels
//     [c*d/16, (c+1)*d/16) of all n streams, i.e. a K-slice of n*d/16 rows of phi.  Its
//     phi slice stays in shared memory for the whole kernel as two bf16 matrices,
//     phi_hi = bf16(phi) and phi_lo = bf16(phi - phi_hi) (16 significant bits, above the
//     TF32 the mixed-precision table asks for), stacked as the 2m rows of the MMA's A
//     operand (K-major, 128-byte swizzle).
//   * Tokens stream through in tiles of NT = 16: one 4-D TMA box per tile copies the
//     CTA's slice of the tile (X read from HBM exactly once) into a ring of stages,
//     ordered as 64-channel atoms a = cb * n + i (channel block cb, stream i).
//   * Six warps issue tcgen05.mma (M = 64 >= 2m, N = 16 tokens, K = 16) over the CTA's
//     K-slice, each into its own TMEM accumulator (the tensor core retires one of these
//     MMAs every ~23 cycles; one issuing warp manages one per ~55).
//   * Four warps copy every stage into TMEM (a ring of stash slots next to the
//     accumulators) while adding the tokens' squares, so a stage is free again as soon
//     as its MMAs are done -- it does not wait for the cluster-wide reduction.
//   * The epilogue ships each token's partial projection to the token's owner CTA
//     (token t of a tile -> CTA t) with one bulk shared-to-peer copy per owner; the
//     owner adds the 16 partials in a fixed order (deterministic, no atomics -- the
//     property the paper's deterministic split-k kernel provides), applies 1/r (RMSNorm
//     after the projection), forms H_pre and sends it to the 16 CTAs.  Sinkhorn (H_res)
//     and H_post run off the critical path in a separate warp, 32 tokens at a time.
//   * Once a tile's H_pre has arrived, four x_in warps read the tile back from TMEM and
//     form x_in for their channels.
//
// Warp roles (672 threads): 0 TMA producer, 1 and 16-20 MMA issuers (warp 1 owns TMEM),
// 2 owner reduction, 3 Sinkhorn / H writer, 4-7 TMEM epilogue, 8-11 stash and sums of
// squares, 12-15 x_in (same TMEM lane quarters as the stash warps).  Every wait on an mbarrier is bounded in time; on expiry the kernel
// records the failing wait in a status word, drains its own copies in flight, frees
// TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.cuh"
#include "tc_ptx.cuh"

namespace mhc {

// Status of the last cluster-kernel launches: 0 = fine, otherwise an OR of the codes of
// the waits that expired (read and cleared by the host through mhc_device_status).
__device__ unsigned int g_pre_tc_status;

namespace tc {

constexpr int S = 16;          // CTAs per cluster
constexpr int NT = 16;         // tokens per tile (MMA N)
constexpr int MAXST = 8;       // max shared-memory stages
constexpr int NMMA = 6;        // MMA-issuing warps = accumulators per buffer
constexpr int NACC = 2;        // TMEM accumulator buffers (tile k uses buffer k % NACC)
constexpr int NSLOT_P = 4;     // receive ring depth (partials in)
constexpr int NSLOT_H = 8;     // H_pre ring depth
constexpr int MAXSTASH = 8;    // TMEM stash slots (tiles of X held for x_in)
constexpr int ACC_COLS = NACC * NMMA * NT;   // TMEM columns of accumulators (192)
constexpr int TMEM_COLS = 512;               // the whole TMEM: one CTA per SM
constexpr int THREADS = (16 + NMMA - 1) * 32;
constexpr int RING = 64;       // logits ring (2 batches of 32 tokens)
constexpr int BATCH = 32;
constexpr int MIN_SMEM = 120 * 1024;          // keeps a second CTA off the SM (TMEM)
constexpr unsigned long long kWaitNs = 1000000000ull;   // 1 s per wait, then give up

template <int N>
struct Cfg {
    static constexpr int M = N * N + 2 * N;       // coefficients per token
    static constexpr int R2 = 2 * M;              // A rows used: [phi_hi^T ; phi_lo^T]
    static constexpr int G = (R2 + 7) / 8;        // 8-row core groups stored per phi atom
    static constexpr int ATOM_PHI = G * 1024;     // bytes of one 64-wide K atom of A
    static constexpr int RECV_D = (R2 + 3) / 4 * 4;
    static constexpr int RECV_STRIDE = RECV_D + 4;          // + sum of squares, padded
    static constexpr int TX_PART = S * (RECV_D * 4 + 4);   // bytes landing per owner / tile
    static constexpr int TX_HPRE = S * 16;                  // H_pre vectors per CTA / tile
    static_assert(R2 <= 64, "A rows must fit M = 64");
};

// instruction descriptor, kind::f16: D fp32, A/B bf16, both K-major, N = 16, M = 64
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
                           ((uint32_t)(64 >> 4) << 24);

// barrier slots (8 bytes each) inside the barrier block
enum : int {
    B_FULL = 0, B_EMPTY = MAXST, B_ACCF = 2 * MAXST, B_ACCE = B_ACCF + NACC,
    B_PART_FULL = B_ACCE + NACC, B_PART_EMPTY = B_PART_FULL + NSLOT_P,
    B_HPRE_FULL = B_PART_EMPTY + NSLOT_P, B_HPRE_EMPTY = B_HPRE_FULL + NSLOT_H,
    B_LG_FULL = B_HPRE_EMPTY + NSLOT_H, B_LG_EMPTY = B_LG_FULL + 2, B_SFULL = B_LG_EMPTY + 2,
    B_SEMPTY = B_SFULL + MAXSTASH, B_STG_READY = B_SEMPTY + MAXSTASH, B_STG_FREE = B_STG_READY + 2,
    B_COUNT = B_STG_FREE + 2
};

// status codes: which wait expired
enum : unsigned {
    E_EMPTY = 1u, E_FULL_MMA = 2u, E_ACCE = 4u, E_ACCF = 8u, E_PART_EMPTY = 16u, E_FULL_SS = 32u,
    E_PART_FULL = 64u, E_HPRE_EMPTY = 128u, E_HPRE_FULL = 512u,
    E_LG_EMPTY = 1024u, E_LG_FULL = 2048u, E_DRAIN = 4096u, E_SFULL = 8192u, E_SEMPTY = 16384u,
    E_STG = 32768u
};

using namespace ptx;

// Bounded wait: true when the phase completed; false when the CTA is aborting or the
// wait expired (then the status word and the CTA's abort flag are set).
template <bool CLUSTER = false>
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned code, bool honour_abort = true) {
    auto try_once = [&]() { return CLUSTER ? mbar_try_cluster(bar, parity) : mbar_try(bar, parity); };
    if (try_once()) return true;
    const uint64_t t0 = gtimer();
    while (true) {
        if (try_once()) return true;
        if (honour_abort && *abort_flag) return false;
        if (gtimer() - t0 > kWaitNs) {
            atomicOr(&g_pre_tc_status, code);
            *abort_flag = 1;
            return false;
        }
    }
}

// ---------------------------------------------------------------- the kernel
template <int N>
__global__ void __launch_bounds__(THREADS, 1)
pre_cluster_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const float* __restrict__ phi,
                      const float* __restrict__ b_pre, const float* __restrict__ b_post,
                      const float* __restrict__ b_res, float a_pre, float a_post, float a_res,
                      int T, int d, float eps, int t_max, __nv_bfloat16* __restrict__ x_in,
                      float* __restrict__ H, float* __restrict__ h_out, int ncb, int nstage)
{
    using C = Cfg<N>;
    constexpr int M = C::M;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* sb = smem_raw + (base - raw);

    const int KA = N * ncb;                 // 64-wide K atoms per CTA (stream x channel block)
    const int cpc = ncb * 64;               // channels per CTA
    const int nchain = KA < NMMA ? KA : NMMA;          // accumulators that receive MMAs
    const int stash_cols = 4 * KA;                     // TMEM columns one tile occupies
    const int nstash = min(MAXSTASH, (TMEM_COLS - ACC_COLS) / stash_cols);
    const uint32_t stage_bytes = (uint32_t)KA * (NT * 128);
    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // shared-memory carve-up (offsets from the 1024-aligned base)
    uint32_t off = 0;
    const uint32_t o_phi = off;  off += (uint32_t)KA * C::ATOM_PHI;
    const uint32_t o_x = off;    off += (uint32_t)nstage * stage_bytes;
    const uint32_t o_recv = off; off += (uint32_t)NSLOT_P * S * C::RECV_STRIDE * 4u;
    const uint32_t o_hpre = off; off += (uint32_t)NSLOT_H * NT * 16u;
    const uint32_t o_ring = off; off += (uint32_t)RING * M * 4u;
    const uint32_t o_stg = off;  off += 2u * NT * C::RECV_D * 4u;    // epilogue staging, 2 tiles
    off = (off + 15u) & ~15u;
    const uint32_t o_bar = off;  off += B_COUNT * 8u;
    const uint32_t o_misc = off;
    float* recv = reinterpret_cast<float*>(sb + o_recv);
    float* hpre = reinterpret_cast<float*>(sb + o_hpre);
    float* ring = reinterpret_cast<float*>(sb + o_ring);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sb + o_misc);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sb + o_misc + 4);
    auto bar = [&](int i) -> uint32_t { return base + o_bar + 8u * (uint32_t)i; };

    const int num_tiles = (T + NT - 1) / NT;
    const int cid = (int)cluster_idx(), ncl = (int)cluster_count();
    const int my_tiles = cid < num_tiles ? (num_tiles - cid + ncl - 1) / ncl : 0;

    // ---------------- set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; ++s) {
            mbar_init(bar(B_FULL + s), 1);
            mbar_init(bar(B_EMPTY + s), NMMA + 4);   // MMA warps' commits + 4 stash warps
        }
        for (int ab = 0; ab < NACC; ++ab) {
            mbar_init(bar(B_ACCF + ab), NMMA);
            mbar_init(bar(B_ACCE + ab), 4);          // 4 epilogue warps
        }
        for (int sl = 0; sl < NSLOT_P; ++sl) {
            mbar_init(bar(B_PART_FULL + sl), 1);
            mbar_init(bar(B_PART_EMPTY + sl), S);    // one arrive per owner CTA
        }
        for (int sl = 0; sl < NSLOT_H; ++sl) {
            mbar_init(bar(B_HPRE_FULL + sl), 1);
            mbar_init(bar(B_HPRE_EMPTY + sl), S * 4);   // 4 stash warps of every CTA
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_LG_FULL + b), 1);
            mbar_init(bar(B_LG_EMPTY + b), 1);
        }
        for (int j = 0; j < MAXSTASH; ++j) {
            mbar_init(bar(B_SFULL + j), 4);      // 4 stash warps wrote the slot
            mbar_init(bar(B_SEMPTY + j), 4);     // 4 x_in warps read it
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_STG_READY + b), 4);  // 4 epilogue warps staged their rows
            mbar_init(bar(B_STG_FREE + b), 4);   // 4 epilogue warps' copies have read it
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), (uint32_t)TMEM_COLS);

    // phi slice -> shared memory as [phi_hi^T ; phi_lo^T] atoms (rows = output columns)
    for (int idx = warp; idx < KA * 8; idx += THREADS / 32) {
        const int a = idx >> 3, j8 = idx & 7;
        const int cb = a / N, i = a - cb * N;              // atom a = cb * n + i
        const int64_t k0 = (int64_t)i * d + (int64_t)rank * cpc + cb * 64 + j8 * 8;
        if (lane < M) {
            float hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float v = __ldg(phi + (k0 + e) * M + lane);
                const __nv_bfloat16 h = __float2bfloat16_rn(v);
                hi[e] = __bfloat162float(h);
                lo[e] = v - hi[e];
            }
            uint8_t* atom = sb + o_phi + (uint32_t)a * C::ATOM_PHI;
            *reinterpret_cast<uint4*>(atom + sw128_off(lane, j8)) = Vec16<__nv_bfloat16>::pack(hi);
            *reinterpret_cast<uint4*>(atom + sw128_off(M + lane, j8)) = Vec16<__nv_bfloat16>::pack(lo);
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int sl = 0; sl < NSLOT_P; ++sl) mbar_arrive_tx(bar(B_PART_FULL + sl), C::TX_PART);
        for (int sl = 0; sl < NSLOT_H; ++sl) mbar_arrive_tx(bar(B_HPRE_FULL + sl), C::TX_HPRE);
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---------------- roles
    if (warp == 0) {
        // TMA producer
        int issued = 0;
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" :: "l"(&tmap_x) : "memory");
            for (int k = 0; k < my_tiles; ++k) {
                const int s = k % nstage, u = k / nstage;
                if (!wait_phase(bar(B_EMPTY + s), (u & 1) ^ 1, abort_flag, E_EMPTY)) break;
                mbar_arrive_tx(bar(B_FULL + s), stage_bytes);
                const int t0 = (cid + k * ncl) * NT;
                // box (64 channels, 16 tokens, n streams, ncb blocks): atoms a = cb * n + i
                tma_load_4d(base + o_x + (uint32_t)s * stage_bytes, &tmap_x, bar(B_FULL + s),
                            0, t0, 0, (int)rank * ncb);
                issued = k + 1;
            }
            // drain: every issued copy has landed before the CTA can leave
            for (int k = issued - 1; k >= 0 && k >= issued - nstage; --k)
                wait_phase(bar(B_FULL + k % nstage), (k / nstage) & 1, abort_flag, E_DRAIN, false);
        }
        __syncwarp();
    } else if (warp == 1 || warp >= 16) {
        // MMA issuers: warp mw issues the K atoms a = mw, mw + nchain, ... into accumulator mw
        const int mw = warp == 1 ? 0 : warp - 15;     // warps 16.. -> 1..
        if (lane == 0) {
            int issued = 0;
            // descriptors advance by adding to the start-address field (16-byte units)
            const uint64_t a_step = (uint64_t)((nchain * C::ATOM_PHI) >> 4);
            const uint64_t b_step = (uint64_t)((nchain * NT * 128) >> 4);
            const uint64_t a_first = sw128_desc(base + o_phi + (uint32_t)mw * C::ATOM_PHI);
            for (int k = 0; k < my_tiles; ++k) {
                const int s = k % nstage, u = k / nstage, ab = k % NACC, ua = k / NACC;
                if (!wait_phase(bar(B_FULL + s), u & 1, abort_flag, E_FULL_MMA)) break;
                if (!wait_phase(bar(B_ACCE + ab), (ua & 1) ^ 1, abort_flag, E_ACCE)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)((ab * NMMA + mw) * NT);
                uint64_t ad = a_first;
                uint64_t bd = sw128_desc(base + o_x + (uint32_t)s * stage_bytes + (uint32_t)mw * (NT * 128));
                uint32_t accumulate = 0;
                for (int a = mw; a < KA && mw < nchain; a += nchain) {
                    mma_bf16(d_tmem, ad, bd, IDESC, accumulate);
                    mma_bf16(d_tmem, ad + 2, bd + 2, IDESC, 1);
                    mma_bf16(d_tmem, ad + 4, bd + 4, IDESC, 1);
                    mma_bf16(d_tmem, ad + 6, bd + 6, IDESC, 1);
                    accumulate = 1;
                    ad += a_step;
                    bd += b_step;
                }
                mma_commit(bar(B_EMPTY + s));
                mma_commit(bar(B_ACCF + ab));
                issued = k + 1;
            }
            if (issued > 0)   // all MMAs complete before TMEM is released
                wait_phase(bar(B_ACCF + (issued - 1) % NACC), ((issued - 1) / NACC) & 1,
                           abort_flag, E_DRAIN, false);
        }
        __syncwarp();
    } else if (warp == 2) {
        // owner: reduce the 16 partials of this CTA's token, broadcast H_pre, queue logits
        const float invK = 1.0f / (float)(N * d);
        // lane j's bias and gate scalar, loaded once
        float bias = 0.f, alpha = 0.f;
        if (lane < N) { bias = __ldg(b_pre + lane); alpha = a_pre; }
        else if (lane < N + N * N) { bias = __ldg(b_res + (lane - N)); alpha = a_res; }
        else if (lane < M) { bias = __ldg(b_post + (lane - N - N * N)); alpha = a_post; }
        for (int k = 0; k < my_tiles; ++k) {
            const int slp = k % NSLOT_P, vp = k / NSLOT_P, slh = k % NSLOT_H, vh = k / NSLOT_H;
            if (!wait_phase<true>(bar(B_PART_FULL + slp), vp & 1, abort_flag, E_PART_FULL)) break;
            const float* rb = recv + slp * S * C::RECV_STRIDE;
            float ss = 0.f;
#pragma unroll
            for (int src = 0; src < S; ++src) ss += rb[src * C::RECV_STRIDE + C::RECV_D];
            float h = 0.f;
            if (lane < M) {
                float hh = 0.f, hl = 0.f;
#pragma unroll
                for (int src = 0; src < S; ++src) {
                    hh += rb[src * C::RECV_STRIDE + lane];
                    hl += rb[src * C::RECV_STRIDE + M + lane];
                }
                h = hh + hl;
            }
            const float inv_r = 1.0f / sqrtf(ss * invK + eps);
            const float z = alpha * (h * inv_r) + bias;
            if (h_out != nullptr && lane < M) {   // the normalised projection, for the backward
                const int64_t tok = (int64_t)(cid + k * ncl) * NT + rank;
                if (tok < T) h_out[tok * M + lane] = h * inv_r;
            }
            const float hp = lane < N ? sigmoid_f32(z) : 0.f;
            float hv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) hv[i] = __shfl_sync(0xffffffffu, hp, i < N ? i : 31);
            __syncwarp();
            // release the receive slot: arm its next phase, then tell the 16 senders
            if (lane == 0) mbar_arrive_tx(bar(B_PART_FULL + slp), C::TX_PART);
            __syncwarp();
            if (lane < S) mbar_arrive_remote(mapa(bar(B_PART_EMPTY + slp), lane));
            // H_pre of this token -> slot slh of every CTA
            if (!wait_phase(bar(B_HPRE_EMPTY + slh), (vh & 1) ^ 1, abort_flag, E_HPRE_EMPTY)) break;
            if (lane < S) {
                const uint32_t dst = smem_u32(hpre + (slh * NT + (int)rank) * 4);
                st_async_v4(mapa(dst, lane), hv[0], N > 1 ? hv[1] : 0.f, N > 2 ? hv[2] : 0.f,
                            N > 3 ? hv[3] : 0.f, mapa(bar(B_HPRE_FULL + slh), lane));
            }
            // [H_pre | res logits | post logits] -> ring for the Sinkhorn warp
            const int bi = k / BATCH, b = bi & 1;
            if ((k % BATCH) == 0 &&
                !wait_phase(bar(B_LG_EMPTY + b), ((bi >> 1) & 1) ^ 1, abort_flag, E_LG_EMPTY)) break;
            if (lane < M) ring[(k % RING) * M + lane] = lane < N ? hp : z;
            __syncwarp();
            if (lane == 0 && ((k % BATCH) == BATCH - 1 || k == my_tiles - 1)) mbar_arrive(bar(B_LG_FULL + b));
        }
    } else if (warp == 3) {
        // Sinkhorn-Knopp (H_res), H_post and the H store, 32 tokens per pass
        const int nb = (my_tiles + BATCH - 1) / BATCH;
        for (int bi = 0; bi < nb; ++bi) {
            const int b = bi & 1;
            if (!wait_phase(bar(B_LG_FULL + b), (bi >> 1) & 1, abort_flag, E_LG_FULL)) break;
            const int k = bi * BATCH + lane;
            if (k < my_tiles) {
                const float* L = ring + (k % RING) * M;
                const int64_t tok = (int64_t)(cid + k * ncl) * NT + rank;
                float out[M];
#pragma unroll
                for (int i = 0; i < N; ++i) out[i] = L[i];
                float Mx[N][N];
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int j = 0; j < N; ++j) Mx[i][j] = expf(L[N + i * N + j]);
                sinkhorn_rounds<N>(Mx, t_max);
#pragma unroll
                for (int i = 0; i < N; ++i)
#pragma unroll
                    for (int j = 0; j < N; ++j) out[N + i * N + j] = Mx[i][j];
#pragma unroll
                for (int i = 0; i < N; ++i) out[N + N * N + i] = 2.0f * sigmoid_f32(L[N + N * N + i]);
                if (tok < T) {
#pragma unroll
                    for (int j = 0; j < M; ++j) H[tok * M + j] = out[j];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_LG_EMPTY + b));
        }
    } else if (warp < 8) {
        // TMEM epilogue: sum the accumulators and stage the tile's partial projections as
        // [token][row]; then warp q bulk-copies tokens 4q..4q+3 to their owner CTAs (one
        // copy of the token's whole row each: 16 copies per tile in all)
        const int q = warp & 3;
        const bool has_rows = 16 * q < C::RECV_D;
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        float* stg0 = reinterpret_cast<float*>(sb + o_stg);
        for (int k = 0; k < my_tiles; ++k) {
            const int ab = k % NACC, ua = k / NACC, slp = k % NSLOT_P, vp = k / NSLOT_P;
            const int b = k & 1, ub = k >> 1;
            if (!wait_phase(bar(B_ACCF + ab), ua & 1, abort_flag, E_ACCF)) break;
            tc_fence_after();
            float dv[16];
            if (has_rows) {
                // accumulators are adjacent 16-column blocks: load two per instruction
#pragma unroll
                for (int t = 0; t < NT; ++t) dv[t] = 0.f;
                for (int c = 0; c < nchain; c += 2) {
                    if (c + 1 < nchain) {
                        float e[32];
                        tmem_ld32(tq + (uint32_t)((ab * NMMA + c) * NT), e);
#pragma unroll
                        for (int t = 0; t < NT; ++t) dv[t] += e[t] + e[NT + t];
                    } else {
                        float e[16];
                        tmem_ld16(tq + (uint32_t)((ab * NMMA + c) * NT), e);
#pragma unroll
                        for (int t = 0; t < NT; ++t) dv[t] += e[t];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_ACCE + ab));
            // stage rows 16q..16q+15 of every token into buffer b
            float* stg = stg0 + b * (NT * C::RECV_D);
            if (!wait_phase(bar(B_STG_FREE + b), (ub & 1) ^ 1, abort_flag, E_STG)) break;
            if (has_rows && lane < 16 && 16 * q + lane < C::RECV_D) {
#pragma unroll
                for (int t = 0; t < NT; ++t) stg[t * C::RECV_D + 16 * q + lane] = dv[t];
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_STG_READY + b));
            if (!wait_phase(bar(B_STG_READY + b), ub & 1, abort_flag, E_STG)) break;
            if (!wait_phase(bar(B_PART_EMPTY + slp), (vp & 1) ^ 1, abort_flag, E_PART_EMPTY)) break;
            if (lane < 4) {
                const int owner = 4 * q + lane;
                const uint32_t dst = base + o_recv + (uint32_t)((slp * S + (int)rank) * C::RECV_STRIDE) * 4u;
                bulk_to_peer(mapa(dst, owner), smem_u32(stg + owner * C::RECV_D), C::RECV_D * 4,
                             mapa(bar(B_PART_FULL + slp), owner));
                // the previous tile's copies (other buffer) have read their source by now
                bulk_wait_read_allbut1();
            }
            __syncwarp();
            if (k > 0 && lane == 0) mbar_arrive(bar(B_STG_FREE + (b ^ 1)));
        }
        if (lane < 4) bulk_wait_all();
    } else if (warp < 12) {
        // stash warps (8-11): thread = (token t, 16-byte chunk u8) = TMEM lane 32q + lane.
        // Per tile: copy the token's chunk of every atom into a TMEM stash slot, add its
        // squares, send the sum to the owner and release the stage.
        const int q = warp & 3;
        const int t = q * 4 + (lane >> 3), u8 = lane & 7;
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        auto stash_col = [&](int k) -> uint32_t { return (uint32_t)(ACC_COLS + (k % nstash) * stash_cols); };
        for (int k = 0; k < my_tiles; ++k) {
            const int s = k % nstage, u = k / nstage, slp = k % NSLOT_P, vp = k / NSLOT_P;
            const int js = k % nstash, us = k / nstash;
            if (!wait_phase(bar(B_SEMPTY + js), (us & 1) ^ 1, abort_flag, E_SEMPTY)) break;
            if (!wait_phase(bar(B_FULL + s), u & 1, abort_flag, E_FULL_SS)) break;
            tc_fence_after();
            const uint8_t* xs = sb + o_x + (uint32_t)s * stage_bytes;
            const uint32_t col = tq + stash_col(k);
            float ss = 0.f;
            for (int a = 0; a < KA; ++a) {
                const uint4 w = *reinterpret_cast<const uint4*>(xs + a * (NT * 128) + sw128_off(t, u8));
                tmem_st4(col + (uint32_t)(4 * a), w);
                float f[8];
                Vec16<__nv_bfloat16>::unpack(w, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
            }
            tmem_wait_st();
            tc_fence_before();
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            ss += __shfl_xor_sync(0xffffffffu, ss, 4);
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_EMPTY + s));
                mbar_arrive(bar(B_SFULL + js));
            }
            if (!wait_phase(bar(B_PART_EMPTY + slp), (vp & 1) ^ 1, abort_flag, E_PART_EMPTY)) break;
            if (u8 == 0) {
                const uint32_t dst = base + o_recv +
                                     (uint32_t)((slp * S + (int)rank) * C::RECV_STRIDE + C::RECV_D) * 4u;
                st_async_f32(mapa(dst, t), ss, mapa(bar(B_PART_FULL + slp), t));
            }
        }
    } else {
        // x_in warps (12-15), same TMEM lanes as the stash warps: once a tile's H_pre has
        // arrived, read its stash slot back and form x_in for this CTA's channels
        const int q = warp & 3;
        const int t = q * 4 + (lane >> 3), u8 = lane & 7;
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        auto stash_col = [&](int k) -> uint32_t { return (uint32_t)(ACC_COLS + (k % nstash) * stash_cols); };
        auto read_map = [&](int j) -> bool {     // x_in for tile j
            const int slh = j % NSLOT_H, vh = j / NSLOT_H;
            if (!wait_phase<true>(bar(B_HPRE_FULL + slh), vh & 1, abort_flag, E_HPRE_FULL)) return false;
            float hp[N];
#pragma unroll
            for (int i = 0; i < N; ++i) hp[i] = hpre[(slh * NT + t) * 4 + i];
            __syncwarp();
            // arm the slot's next phase: it cannot complete before all four stash warps of
            // every CTA (this one's included) have released this phase below
            if (warp == 12 && lane == 0) mbar_arrive_tx(bar(B_HPRE_FULL + slh), C::TX_HPRE);
            __syncwarp();
            if (lane < S) mbar_arrive_remote(mapa(bar(B_HPRE_EMPTY + slh), lane));
            const int64_t tok = (int64_t)(cid + j * ncl) * NT + t;
            const uint32_t col = tq + stash_col(j);
            tc_fence_after();
            for (int cb = 0; cb < ncb; ++cb) {
                float acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    const uint4 w = tmem_ld4(col + (uint32_t)(4 * (cb * N + i)));
                    float f[8];
                    Vec16<__nv_bfloat16>::unpack(w, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] = fmaf(hp[i], f[e], acc[e]);
                }
                if (tok < T)
                    st_v4(x_in + tok * d + (int)rank * cpc + cb * 64 + u8 * 8, Vec16<__nv_bfloat16>::pack(acc));
            }
            return true;
        };
        for (int j = 0; j < my_tiles; ++j) {
            const int js = j % nstash, us = j / nstash;
            if (!wait_phase(bar(B_SFULL + js), us & 1, abort_flag, E_SFULL)) break;
            if (!read_map(j)) break;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SEMPTY + js));
        }
    }

    // ---------------- tear-down: no peer touches this CTA's shared memory after this
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    bool ok = false;
    int nstage = 0, smem = 0, max_clusters = 0;
};

template <int N>
int smem_bytes(int ncb, int nstage) {
    using C = Cfg<N>;
    const int KA = N * ncb;
    int off = KA * C::ATOM_PHI + nstage * KA * NT * 128 + NSLOT_P * S * C::RECV_STRIDE * 4 +
              NSLOT_H * NT * 16 + RING * C::M * 4 + 2 * NT * C::RECV_D * 4;
    off = (off + 15) & ~15;
    off += B_COUNT * 8 + 16;
    off += 1024;         // alignment slack of the dynamic shared-memory base
    return off < MIN_SMEM ? MIN_SMEM : off;
}

template <int N>
Plan make_plan(int ncb) {
    Plan p;
    DeviceInfo di;
    if (device_info(&di) != cudaSuccess || di.cc_major != 10 || di.cc_minor != 0) return p;
    int ns = MAXST;
    while (ns >= 2 && smem_bytes<N>(ncb, ns) > di.max_smem_optin) --ns;
    if (ns < 2) return p;
    // the last phi atom's 64-row MMA read runs (8 - G) KB past the phi region: stay inside
    if (smem_bytes<N>(ncb, ns) - 1024 < N * ncb * Cfg<N>::ATOM_PHI + (8 - Cfg<N>::G) * 1024) return p;
    const int smem = smem_bytes<N>(ncb, ns);
    auto kern = pre_cluster_tc_kernel<N>;
    // the limit is a property of the function, shared by every plan of this n: set the device's
    // maximum so that no plan's launch is refused after another plan was made
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, di.max_smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return p;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S * 8);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = S;
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
    p.smem = smem;
    p.max_clusters = nc;
    return p;
}

// plans cached per (device, n, channel blocks per CTA)
Plan get_plan(int n, int ncb) {
    static std::mutex mu;
    static Plan cache[64][5][5];
    static bool have[64][5][5] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || n < 1 || n > 4 || ncb < 1 || ncb > 4) {
        cudaGetLastError();
        return Plan{};
    }
    std::lock_guard<std::mutex> lk(mu);
    if (!have[dev][n][ncb]) {
        Plan p;
        switch (n) {
            case 1: p = make_plan<1>(ncb); break;
            case 2: p = make_plan<2>(ncb); break;
            case 3: p = make_plan<3>(ncb); break;
            case 4: p = make_plan<4>(ncb); break;
        }
        cache[dev][n][ncb] = p;
        have[dev][n][ncb] = true;
    }
    return cache[dev][n][ncb];
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
cudaError_t launch_n(const PreArgs& a, const Plan& p, int ncb) {
    // X viewed as 4-D: (channel within a 64-block: 64, token: T, stream: n, block: d/64);
    // one box (64, 16, n, d/1024) is a CTA's whole slice of a 16-token tile
    CUtensorMap map;
    const cuuint64_t dims[4] = {64, (cuuint64_t)a.T, (cuuint64_t)N, (cuuint64_t)(a.d / 64)};
    const cuuint64_t strides[3] = {(cuuint64_t)N * a.d * 2, (cuuint64_t)a.d * 2, 128};
    const cuuint32_t box[4] = {64, NT, (cuuint32_t)N, (cuuint32_t)ncb};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(a.X), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int num_tiles = (int)((a.T + NT - 1) / NT);
    const int ncl = num_tiles < p.max_clusters ? num_tiles : p.max_clusters;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ncl * S));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = S;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, pre_cluster_tc_kernel<N>, map, a.phi, a.b_pre, a.b_post, a.b_res,
                              a.a_pre, a.a_post, a.a_res, (int)a.T, a.d, a.eps, a.t_max,
                              static_cast<__nv_bfloat16*>(a.x_in), a.H, a.h_out, ncb, p.nstage);
}

}  // namespace tc

bool pre_cluster_tc_shape_ok(int64_t T, int n, int d, DType dt) {
    return dt == BF16 && n >= 1 && n <= 4 && d >= 1024 && d <= 4096 && d % 1024 == 0 && T >= 1 &&
           T < ((int64_t)1 << 31) - tc::NT;
}

bool pre_cluster_tc_device_ok(int n, int d) {
    if (n < 1 || n > 4 || d % 1024 != 0 || d > 4096) return false;
    return tc::get_plan(n, d / 1024).ok;
}

cudaError_t launch_pre_cluster_tc(const PreArgs& a) {
    const int ncb = a.d / 1024;
    const tc::Plan p = tc::get_plan(a.n, ncb);
    if (!p.ok) return cudaErrorNotSupported;
    switch (a.n) {
        case 1: return tc::launch_n<1>(a, p, ncb);
        case 2: return tc::launch_n<2>(a, p, ncb);
        case 3: return tc::launch_n<3>(a, p, ncb);
        case 4: return tc::launch_n<4>(a, p, ncb);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t pre_cluster_tc_status(unsigned* out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_pre_tc_status, sizeof(unsigned));
    if (e != cudaSuccess) return e;
    if (clear && *out) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_pre_tc_status, &zero, sizeof(unsigned));
    }
    return e;
}

}  // namespace mhc
