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
//   * Tokens stream through in tiles of NT = 16: TMA copies each CTA's slice of the
//     tile's rows (X read from HBM exactly once) into a ring of shared-memory stages.
//   * One thread issues tcgen05.mma (M = 64 >= 2m, N = 16 tokens, K = 16) over the
//     CTA's K-slice into a TMEM accumulator: the partial projection of 16 tokens.
//   * Partials go to the token's owner CTA (token t of a tile -> CTA t) by st.async
//     into its shared memory, with the partial sum of squares; the owner adds the 16
//     partials in a fixed order (deterministic, no atomics -- the property the paper's
//     deterministic split-k kernel provides), applies 1/r (RMSNorm after the
//     projection), forms H_pre and broadcasts it to the 16 CTAs.
//   * Every CTA then computes x_in for its channels from the X tile still in shared
//     memory and stores it.  Sinkhorn (H_res) and H_post run off the critical path in a
//     separate warp, 32 tokens at a time, and write the coefficient block H.
//
// Warp roles (512 threads): 0 TMA producer, 1 MMA issuer (+ TMEM owner), 2 owner
// reduction, 3 Sinkhorn / H writer, 4-7 TMEM epilogue, 8-11 sum of squares, 12-15 x_in.
// Issuing a tcgen05.mma costs the issuing thread ~100 cycles whatever the shape, so four
// warps issue a tile's MMAs, each into its own TMEM accumulator; the epilogue adds the
// accumulators in a fixed order and ships each owner its rows with one bulk
// shared-to-shared copy.
// Every wait on an mbarrier is bounded in time; on expiry the kernel records the failing
// wait in a status word, drains its own copies in flight, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "launch.cuh"

namespace mhc {

// Status of the last cluster-kernel launches: 0 = fine, otherwise an OR of the codes of
// the waits that expired (read and cleared by the host through mhc_device_status).
__device__ unsigned int g_pre_tc_status;

namespace tc {

constexpr int S = 16;          // CTAs per cluster
constexpr int NT = 16;         // tokens per tile (MMA N)
constexpr int MAXST = 8;       // max shared-memory stages
constexpr int NMMA = 4;        // warps issuing tcgen05.mma (issue cost is per thread)
constexpr int THREADS = 512 + 32 * (NMMA - 1);
constexpr int NSLOT = 4;       // depth of the cross-CTA rings (partials in, H_pre out)
constexpr int NACC = 2;        // TMEM accumulator buffers (tile k uses buffer k % NACC)
constexpr int MAXCHAIN = NMMA; // one accumulation chain per MMA warp
constexpr int RING = 64;       // logits ring (2 batches of 32 tokens)
constexpr int BATCH = 32;
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
    B_FULL = 0, B_EMPTY = MAXST, B_ACCF = 2 * MAXST, B_ACCE = 3 * MAXST,
    B_PART_FULL = 4 * MAXST, B_PART_EMPTY = B_PART_FULL + NSLOT,
    B_HPRE_FULL = B_PART_EMPTY + NSLOT, B_HPRE_EMPTY = B_HPRE_FULL + NSLOT,
    B_LG_FULL = B_HPRE_EMPTY + NSLOT, B_LG_EMPTY = B_LG_FULL + 2, B_COUNT = B_LG_EMPTY + 2
};

// status codes: which wait expired
enum : unsigned {
    E_EMPTY = 1u, E_FULL_MMA = 2u, E_ACCE = 4u, E_ACCF = 8u, E_PART_EMPTY = 16u, E_FULL_SS = 32u,
    E_PART_FULL = 64u, E_HPRE_EMPTY = 128u, E_FULL_XIN = 256u, E_HPRE_FULL = 512u,
    E_LG_EMPTY = 1024u, E_LG_FULL = 2048u, E_DRAIN = 4096u
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r; asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r)); return r;
}
__device__ __forceinline__ uint32_t cluster_idx() {
    uint32_t r; asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r)); return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r; asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r)); return r;
}
__device__ __forceinline__ uint64_t gtimer() {
    uint64_t t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}
// Arrive on an mbarrier of another CTA of the cluster (shared::cluster address).  Used
// only to say "this buffer may be overwritten": every value read from the buffer has
// been consumed by an instruction before the arrive, so no release fence is needed (a
// release here would also wait for this warp's earlier global stores).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cbar) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" :: "r"(cbar) : "memory");
}
// CTA-scope acquire: barriers completed by this CTA's own threads, TMA or tensor cores
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// cluster-scope acquire: barriers whose phase completes with data st.async'd by peers
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_async_v4(uint32_t raddr, float a, float b, float c, float d,
                                            uint32_t rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
                 :: "r"(raddr), "f"(a), "f"(b), "f"(c), "f"(d), "r"(rbar) : "memory");
}
__device__ __forceinline__ void st_async_f32(uint32_t raddr, float a, uint32_t rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];"
                 :: "r"(raddr), "f"(a), "r"(rbar) : "memory");
}
// bulk copy of `bytes` (multiple of 16) from this CTA's shared memory into a peer's,
// completing `bytes` of transaction count on the peer's mbarrier
__device__ __forceinline__ void bulk_to_peer(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes,
                                             uint32_t rbar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst_cluster), "r"(src_cta), "r"(bytes), "r"(rbar) : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_allbut1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3, %4}], [%5];"
                 :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(dst_smem), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(IDESC), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns; waits for the load before returning
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr) : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// byte offset of 16-byte chunk j of row r inside a 128-byte-swizzled block of 8-row groups
__device__ __forceinline__ uint32_t sw128_off(int r, int j) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

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
                      float* __restrict__ H, int ncb, int nstage, int nchain, int tmem_cols)
{
    using C = Cfg<N>;
    constexpr int M = C::M;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* sb = smem_raw + (base - raw);

    const int KA = N * ncb;                 // 64-wide K atoms per CTA (stream x channel block)
    const int cpc = ncb * 64;               // channels per CTA
    const uint32_t stage_bytes = (uint32_t)KA * (NT * 128);
    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // shared-memory carve-up (offsets from the 1024-aligned base)
    uint32_t off = 0;
    const uint32_t o_phi = off;  off += (uint32_t)KA * C::ATOM_PHI;
    const uint32_t o_x = off;    off += (uint32_t)nstage * stage_bytes;
    const uint32_t o_recv = off; off += (uint32_t)NSLOT * S * C::RECV_STRIDE * 4u;
    const uint32_t o_hpre = off; off += (uint32_t)NSLOT * NT * 16u;
    const uint32_t o_ring = off; off += (uint32_t)RING * M * 4u;
    const uint32_t o_stg = off;  off += 4u * 2u * NT * 16u * 4u;     // epilogue staging, per warp x2
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
            mbar_init(bar(B_EMPTY + s), NMMA + 8);   // MMA warps + 4 sum-of-squares + 4 x_in
        }
        for (int ab = 0; ab < NACC; ++ab) {
            mbar_init(bar(B_ACCF + ab), NMMA);
            mbar_init(bar(B_ACCE + ab), 4);       // 4 epilogue warps
        }
        for (int sl = 0; sl < NSLOT; ++sl) {
            mbar_init(bar(B_PART_FULL + sl), 1);
            mbar_init(bar(B_PART_EMPTY + sl), S);        // one arrive per owner CTA
            mbar_init(bar(B_HPRE_FULL + sl), 1);
            mbar_init(bar(B_HPRE_EMPTY + sl), S * 4);    // 4 x_in warps of every CTA
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_LG_FULL + b), 1);
            mbar_init(bar(B_LG_EMPTY + b), 1);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), (uint32_t)tmem_cols);

    // phi slice -> shared memory as [phi_hi^T ; phi_lo^T] atoms (rows = output columns)
    for (int idx = warp; idx < KA * 8; idx += THREADS / 32) {
        const int a = idx >> 3, j8 = idx & 7;
        const int i = a / ncb, cb = a - i * ncb;
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
        for (int sl = 0; sl < NSLOT; ++sl) {
            mbar_arrive_tx(bar(B_PART_FULL + sl), C::TX_PART);
            mbar_arrive_tx(bar(B_HPRE_FULL + sl), C::TX_HPRE);
        }
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
                const uint32_t dst = base + o_x + (uint32_t)s * stage_bytes;
                for (int a = 0; a < KA; ++a) {
                    const int i = a / ncb, cb = a - i * ncb;
                    tma_load_3d(dst + (uint32_t)a * (NT * 128), &tmap_x, bar(B_FULL + s),
                                (int)rank * cpc + cb * 64, i, t0);
                }
                issued = k + 1;
            }
            // drain: every issued copy has landed before the CTA can leave
            for (int k = issued - 1; k >= 0 && k >= issued - nstage; --k)
                wait_phase(bar(B_FULL + k % nstage), (k / nstage) & 1, abort_flag, E_DRAIN, false);
        }
        __syncwarp();
    } else if (warp == 1 || warp >= 16) {
        // MMA issuers: warp mw issues the K atoms a = mw, mw + nchain, ... into chain mw
        const int mw = warp == 1 ? 0 : warp - 15;
        if (lane == 0) {
            int issued = 0;
            for (int k = 0; k < my_tiles; ++k) {
                const int s = k % nstage, u = k / nstage, ab = k % NACC, ua = k / NACC;
                if (!wait_phase(bar(B_FULL + s), u & 1, abort_flag, E_FULL_MMA)) break;
                if (!wait_phase(bar(B_ACCE + ab), (ua & 1) ^ 1, abort_flag, E_ACCE)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(ab * nchain * NT);
                const uint32_t xs = base + o_x + (uint32_t)s * stage_bytes;
                for (int a = mw; a < KA && mw < nchain; a += nchain) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = sw128_desc(base + o_phi + (uint32_t)a * C::ATOM_PHI + kk * 32);
                        const uint64_t bd = sw128_desc(xs + (uint32_t)a * (NT * 128) + kk * 32);
                        mma_bf16(d_tmem + (uint32_t)(mw * NT), ad, bd, (a != mw) || kk);
                    }
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
        for (int k = 0; k < my_tiles; ++k) {
            const int sl = k % NSLOT, v = k / NSLOT;
            if (!wait_phase<true>(bar(B_PART_FULL + sl), v & 1, abort_flag, E_PART_FULL)) break;
            const float* rb = recv + sl * S * C::RECV_STRIDE;
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
            float z = 0.f;
            if (lane < N) z = a_pre * (h * inv_r) + __ldg(b_pre + lane);
            else if (lane < N + N * N) z = a_res * (h * inv_r) + __ldg(b_res + (lane - N));
            else if (lane < M) z = a_post * (h * inv_r) + __ldg(b_post + (lane - N - N * N));
            const float hp = lane < N ? sigmoid_f32(z) : 0.f;
            float hv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) hv[i] = __shfl_sync(0xffffffffu, hp, i < N ? i : 31);
            __syncwarp();
            // release the receive slot: arm its next phase, then tell the 16 senders
            if (lane == 0) mbar_arrive_tx(bar(B_PART_FULL + sl), C::TX_PART);
            __syncwarp();
            if (lane < S) mbar_arrive_remote(mapa(bar(B_PART_EMPTY + sl), lane));
            // H_pre of this token -> slot sl of every CTA
            if (!wait_phase(bar(B_HPRE_EMPTY + sl), (v & 1) ^ 1, abort_flag, E_HPRE_EMPTY)) break;
            if (lane < S) {
                const uint32_t dst = smem_u32(hpre + (sl * NT + (int)rank) * 4);
                st_async_v4(mapa(dst, lane), hv[0], N > 1 ? hv[1] : 0.f, N > 2 ? hv[2] : 0.f,
                            N > 3 ? hv[3] : 0.f, mapa(bar(B_HPRE_FULL + sl), lane));
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
        // TMEM epilogue: sum the accumulation chains, stage this warp's 16 rows of the
        // tile's partial projections, and bulk-copy token t's rows to owner CTA t
        const int q = warp & 3;
        const bool has_rows = 16 * q < C::RECV_D;
        const uint32_t nbytes = (uint32_t)min(16, C::RECV_D - 16 * q) * 4u;
        float* stg = reinterpret_cast<float*>(sb + o_stg) + q * (2 * NT * 16);
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        for (int k = 0; k < my_tiles; ++k) {
            const int ab = k % NACC, ua = k / NACC, sl = k % NSLOT, v = k / NSLOT;
            if (!wait_phase(bar(B_ACCF + ab), ua & 1, abort_flag, E_ACCF)) break;
            tc_fence_after();
            float dv[16];
            if (has_rows) {
                tmem_ld16(tq + (uint32_t)(ab * nchain * NT), dv);
                for (int c = 1; c < nchain; ++c) {
                    float e[16];
                    tmem_ld16(tq + (uint32_t)((ab * nchain + c) * NT), e);
#pragma unroll
                    for (int t = 0; t < NT; ++t) dv[t] += e[t];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_ACCE + ab));
            if (!has_rows) continue;
            float* sbuf = stg + (k & 1) * (NT * 16);
            if (lane < NT) bulk_wait_read_allbut1();     // copies out of sbuf two tiles ago done
            __syncwarp();
            if (lane < 16) {
#pragma unroll
                for (int t = 0; t < NT; ++t) sbuf[t * 16 + lane] = dv[t];
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (!wait_phase(bar(B_PART_EMPTY + sl), (v & 1) ^ 1, abort_flag, E_PART_EMPTY)) break;
            if (lane < NT) {
                const uint32_t dst = base + o_recv +
                                     (uint32_t)((sl * S + (int)rank) * C::RECV_STRIDE + 16 * q) * 4u;
                bulk_to_peer(mapa(dst, lane), smem_u32(sbuf + lane * 16), nbytes,
                             mapa(bar(B_PART_FULL + sl), lane));
            }
        }
        if (lane < NT) bulk_wait_all();
    } else if (warp < 12) {
        // sum of squares of this CTA's slice of every token of the tile -> owners
        const int t = (warp - 8) * 4 + (lane >> 3), u8 = lane & 7;
        for (int k = 0; k < my_tiles; ++k) {
            const int s = k % nstage, u = k / nstage, sl = k % NSLOT, v = k / NSLOT;
            if (!wait_phase(bar(B_FULL + s), u & 1, abort_flag, E_FULL_SS)) break;
            const uint8_t* xs = sb + o_x + (uint32_t)s * stage_bytes;
            float ss = 0.f;
            for (int a = 0; a < KA; ++a) {
                const uint4 w = *reinterpret_cast<const uint4*>(xs + a * (NT * 128) + sw128_off(t, u8));
                float f[8];
                Vec16<__nv_bfloat16>::unpack(w, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            ss += __shfl_xor_sync(0xffffffffu, ss, 4);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_EMPTY + s));
            if (!wait_phase(bar(B_PART_EMPTY + sl), (v & 1) ^ 1, abort_flag, E_PART_EMPTY)) break;
            if (u8 == 0) {
                const uint32_t dst = base + o_recv +
                                     (uint32_t)((sl * S + (int)rank) * C::RECV_STRIDE + C::RECV_D) * 4u;
                st_async_f32(mapa(dst, t), ss, mapa(bar(B_PART_FULL + sl), t));
            }
        }
    } else {
        // x_in = sum_i H_pre[i] X_i for this CTA's channels, from the tile in shared memory
        const int t = (warp - 12) * 4 + (lane >> 3), u8 = lane & 7;
        const int coff = (int)rank * cpc + (u8 << 3);
        for (int k = 0; k < my_tiles; ++k) {
            const int s = k % nstage, u = k / nstage, sl = k % NSLOT, v = k / NSLOT;
            const int64_t tok = (int64_t)(cid + k * ncl) * NT + t;
            if (!wait_phase(bar(B_FULL + s), u & 1, abort_flag, E_FULL_XIN)) break;
            if (!wait_phase<true>(bar(B_HPRE_FULL + sl), v & 1, abort_flag, E_HPRE_FULL)) break;
            float hp[N];
#pragma unroll
            for (int i = 0; i < N; ++i) hp[i] = hpre[(sl * NT + t) * 4 + i];
            const uint8_t* xs = sb + o_x + (uint32_t)s * stage_bytes;
            for (int cb = 0; cb < ncb; ++cb) {
                float acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
                for (int i = 0; i < N; ++i) {
                    const uint4 w = *reinterpret_cast<const uint4*>(
                        xs + (i * ncb + cb) * (NT * 128) + sw128_off(t, u8));
                    float f[8];
                    Vec16<__nv_bfloat16>::unpack(w, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] = fmaf(hp[i], f[e], acc[e]);
                }
                if (tok < T) st_v4(x_in + tok * d + coff + cb * 64, Vec16<__nv_bfloat16>::pack(acc));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_EMPTY + s));
            if (warp == 12 && lane == 0) mbar_arrive_tx(bar(B_HPRE_FULL + sl), C::TX_HPRE);
            __syncwarp();
            if (lane < S) mbar_arrive_remote(mapa(bar(B_HPRE_EMPTY + sl), lane));
        }
    }

    // ---------------- tear-down: no peer touches this CTA's shared memory after this
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)tmem_cols);
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    bool ok = false;
    int nstage = 0, smem = 0, max_clusters = 0, nchain = 0, tmem_cols = 0;
};

template <int N>
int smem_bytes(int ncb, int nstage) {
    using C = Cfg<N>;
    const int KA = N * ncb;
    int off = KA * C::ATOM_PHI + nstage * KA * NT * 128 + NSLOT * S * C::RECV_STRIDE * 4 +
              NSLOT * NT * 16 + RING * C::M * 4 + 4 * 2 * NT * 16 * 4;
    off = (off + 15) & ~15;
    off += B_COUNT * 8 + 16;
    return off + 1024;   // alignment slack of the dynamic shared-memory base
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
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
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
    const int nchain = N * ncb < MAXCHAIN ? N * ncb : MAXCHAIN;   // chains that receive MMAs
    int cols = 32;
    while (cols < NACC * nchain * NT) cols <<= 1;     // <= 256: two CTAs per SM never block
    p.ok = true;
    p.nstage = ns;
    p.smem = smem;
    p.max_clusters = nc;
    p.nchain = nchain;
    p.tmem_cols = cols;
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
    // X viewed as 3-D: (channel c: d, stream i: n, token t: T); box = 64 channels x 1 x 16 tokens
    CUtensorMap map;
    const cuuint64_t dims[3] = {(cuuint64_t)a.d, (cuuint64_t)N, (cuuint64_t)a.T};
    const cuuint64_t strides[2] = {(cuuint64_t)a.d * 2, (cuuint64_t)N * a.d * 2};
    const cuuint32_t box[3] = {64, 1, NT};
    const cuuint32_t estr[3] = {1, 1, 1};
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.X), dims, strides,
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
                              static_cast<__nv_bfloat16*>(a.x_in), a.H, ncb, p.nstage, p.nchain,
                              p.tmem_cols);
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
