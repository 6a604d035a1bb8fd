// pre_tc.cu -- the mHC pre stage on B200 tensor cores: X crosses HBM once.
//
// What it computes is the pre stage of "DeepSeek-V4/mhc" (equations rmsnorm, a/b/c-tilde,
// gate, sinkhorn-init, sinkhorn) and the read map H_pre x_l of the slavadubrov.com Eq. 3;
// see include/mhc.h.  How, on sm_100a:
//
//   * A cluster of S = 16 CTAs splits the flattened K = n*d axis of the projection: CTA r
//     owns a contiguous run of 64-channel atoms of vec(X_t).  Its slice of phi stays in
//     shared memory for the whole kernel as the MMA's B operand, N = 2m rows
//     [phi_hi^T ; phi_lo^T] with phi_hi = bf16(phi), phi_lo = bf16(phi - phi_hi) (16
//     significant bits, above the TF32 the mixed-precision table asks for), K-major,
//     128-byte swizzle.
//   * Tokens stream through in tiles of NT = 64 (the MMA's M): one 3-D TMA box per stage
//     copies SA = 4 atoms of 64 tokens (32 KB; large boxes are what lets one SM's TMA
//     stream keep up with its share of HBM).  Two warps issue tcgen05.mma (M = 64,
//     N = 2m, K = 16), atoms j, j + 2 of a stage from issuer j, each into its own TMEM
//     accumulator (three buffers, so the MMAs of the next tiles do not wait for the
//     epilogue).
//   * The same four warps that read each stage for the tokens' sums of squares read the
//     accumulators back (token t in TMEM lane 32 (t / 16) + t % 16), add hi + lo, and ship
//     each token's partial projection and partial sum of squares to the token's owner CTA
//     (local token t -> CTA t % 16) with one bulk shared-to-peer copy per owner.
//   * The owner adds the 16 partials in a fixed order (deterministic, no atomics -- the
//     property the paper's deterministic split-k provides, without split buffers in
//     HBM), applies 1/r (RMSNorm after the projection) and sends H_pre to all 16 CTAs.
//     A separate warp runs Sinkhorn (H_res) and H_post and writes H, one token per lane,
//     32 tokens (8 tiles) per pass, off the critical path.  (The HC comparison maps take
//     b + alpha tanh(h / r) for every coefficient instead.)
//   * Seven warps form x_in for the CTA's share of the d channels once a tile's H_pre has
//     arrived, re-reading that tile of X with plain loads: the tile was loaded moments
//     before, so those reads hit L2 (the whole GPU keeps a few tiles per cluster, tens of
//     MB, in flight) and X still crosses HBM once.
//
// Warp roles (512 threads): 0 TMA producer and TMEM owner, 1 owner reduction and H_pre,
// 2-3 MMA issuers, 4-7 sums of squares and accumulator epilogue (TMEM lane quarters 0-3),
// 8-14 x_in, 15 Sinkhorn and the H store.  Every wait on an mbarrier is bounded in time; on expiry
// the kernel records the failing wait in a status word, drains its own copies in
// flight, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "launch.cuh"
#include "tc_ptx.cuh"

namespace mhc {

// Status of the tensor-core pre kernel's bounded waits since the last read: 0 = fine,
// otherwise an OR of the codes of the waits that expired (mhc_device_status).
__device__ unsigned int g_pre_tc_status;

namespace tc {

constexpr int S = 16;              // CTAs per cluster
constexpr int NT = 64;             // tokens per tile = MMA M
constexpr int SA = 4;              // 64-channel atoms per stage (TMA box depth)
constexpr int NMMA = 2;            // MMA issuers: atom j of a stage goes to issuer j % NMMA
constexpr int NACC = 3;            // accumulator buffers (tile k -> buffer k % NACC)
constexpr int ACC_STRIDE = 64;     // TMEM columns per accumulator
constexpr int NSLOT_P = 2;         // partial-projection receive slots
constexpr int NSLOT_H = 2;         // H_pre receive slots
constexpr int TPO = NT / S;        // tokens per owner per tile
constexpr int MAXST = 4;           // max X stages
constexpr int PF = 0;              // stages of X prefetched into L2 ahead of their load (measured: none is best)
constexpr int NXW = 7;             // x_in warps
constexpr int SK_WARP = 8 + NXW;   // Sinkhorn warp
constexpr int BATCH = 32;          // tokens per Sinkhorn pass (one per lane)
constexpr int RING = 2 * BATCH;    // logit ring: two passes
constexpr int XU = 2;              // x_in tasks in flight per thread (more slows the X stream: 5 took 7 % longer)
constexpr int NWARPS = 16;         // 4 warps per scheduler partition: up to 128 registers
constexpr int THREADS = NWARPS * 32;
constexpr int TMEM_COLS = 512;
constexpr int STAGE_BYTES = SA * NT * 128;      // 32 KB
constexpr unsigned long long kWaitNs = 1000000000ull;   // 1 s per wait, then give up

static_assert(SA % NMMA == 0, "every issuer gets the same atoms of a full stage");
static_assert(BATCH % TPO == 0, "a Sinkhorn pass holds whole tiles");
static_assert(BATCH == 32, "the Sinkhorn warp takes one token of a pass per lane");
static_assert(SK_WARP + 1 == NWARPS && NMMA == 2, "warp roles fill the block");
static_assert(NACC * NMMA * ACC_STRIDE <= TMEM_COLS, "accumulators fit TMEM");

template <int N>
struct Cfg {
    static constexpr int M = N * N + 2 * N;        // coefficients per token
    static constexpr int NB = (2 * M + 7) / 8 * 8; // MMA N: [hi | lo] rows, padded to 8
    static constexpr int PHI_ATOM = NB / 8 * 1024; // bytes of one atom of the B operand
    static constexpr int W = M + 1;                // floats per token sent to its owner
    static constexpr int PART = TPO * W;           // floats per (source CTA, owner) block
    static constexpr int TX_PART = S * PART * 4;   // bytes landing per owner and tile
    static constexpr int TX_HPRE = NT * 16;        // H_pre bytes landing per CTA and tile
    static_assert(NB <= ACC_STRIDE, "an accumulator fits its TMEM columns");
    static_assert((PART * 4) % 16 == 0, "bulk copies move multiples of 16 bytes");
};

// instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, M = 64, N = nb
__host__ __device__ constexpr uint32_t idesc_m64(int nb) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(nb >> 3) << 17) | ((uint32_t)(64 >> 4) << 24);
}

enum : int {
    B_FULL = 0, B_EMPTY = MAXST, B_ACCF = 2 * MAXST, B_ACCE = B_ACCF + NACC,
    B_PFULL = B_ACCE + NACC, B_PEMPTY = B_PFULL + NSLOT_P, B_HFULL = B_PEMPTY + NSLOT_P,
    B_HEMPTY = B_HFULL + NSLOT_H, B_DRAIN = B_HEMPTY + NSLOT_H, B_STG_FREE = B_DRAIN + NMMA,
    B_STG_READY = B_STG_FREE + 2, B_XDONE = B_STG_READY + 1, B_LG_FULL = B_XDONE + NSLOT_H,
    B_LG_EMPTY = B_LG_FULL + 2, B_COUNT = B_LG_EMPTY + 2
};

// status codes: which wait expired
enum : unsigned {
    E_EMPTY = 1u, E_FULL_MMA = 2u, E_ACCE = 4u, E_ACCF = 8u, E_PEMPTY = 16u, E_FULL_SS = 32u,
    E_PFULL = 64u, E_HEMPTY = 128u, E_HFULL = 256u, E_DRAIN = 512u, E_STG = 1024u, E_XDONE = 2048u,
    E_LG_EMPTY = 4096u, E_LG_FULL = 8192u
};

using namespace ptx;

struct Waiter {
    volatile int* abort_flag;
    unsigned long long limit_ns;
    // Bounded wait: true when the phase completed; false when the CTA is aborting or the
    // wait expired (then the status word and the CTA's abort flag are set).
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
                atomicOr(&g_pre_tc_status, code);
                *abort_flag = 1;
                return false;
            }
        }
    }
};

// TMEM -> registers without waiting (32 lanes x 8 or 16 consecutive columns); the registers
// are valid only after tmem_wait_regs on them
template <int W>
__device__ __forceinline__ void tmem_ld_nowait(uint32_t taddr, uint32_t* r);
template <>
__device__ __forceinline__ void tmem_ld_nowait<8>(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_nowait<16>(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr) : "memory");
}
// Wait for this thread's TMEM loads; the 8 registers are operands, so no use of them can be
// scheduled before the wait
__device__ __forceinline__ void tmem_wait_regs8(uint32_t* r) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]) :: "memory");
}

// streaming 16-byte read of X for the read map: the tile's last use, so L2 may drop it
__device__ __forceinline__ uint4 ld_last_use_v4(const void* p, uint64_t pol) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p), "l"(pol));
    return r;
}

struct Maps {
    CUtensorMap box[SA];           // box[j]: j + 1 atoms of NT tokens
};

// ---------------------------------------------------------------- the kernel
template <int N>
__global__ void __launch_bounds__(THREADS, 1)
pre_tc_kernel(const __grid_constant__ Maps maps, const __nv_bfloat16* __restrict__ X,
              const float* __restrict__ phi, const float* __restrict__ b_pre,
              const float* __restrict__ b_post, const float* __restrict__ b_res, float a_pre,
              float a_post, float a_res, int T, int d, float eps, int t_max,
              __nv_bfloat16* __restrict__ x_in, float* __restrict__ H, float* __restrict__ h_out,
              int ka_total, int ka_max, int nstage, int stop_tile, unsigned long long wait_ns, int hc)
{
    using C = Cfg<N>;
    constexpr int M = C::M, NB = C::NB, W = C::W;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* sb = smem_raw + (base - raw);

    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's atoms [a_lo, a_lo + ka) of the n*d/64 atoms of vec(X_t)
    const int a_lo = (int)(((int64_t)rank * ka_total) / S);
    const int ka = (int)((((int64_t)rank + 1) * ka_total) / S) - a_lo;
    const int nchain = ka < NMMA ? ka : NMMA;        // accumulators that receive MMAs
    // this CTA's x_in channels: 8-channel chunks [c_lo, c_lo + nch)
    const int nchunks = d >> 3;
    const int c_lo = (int)(((int64_t)rank * nchunks) / S);
    const int nch = (int)((((int64_t)rank + 1) * nchunks) / S) - c_lo;

    // shared-memory carve-up (offsets from the 1024-aligned base)
    uint32_t off = 0;
    const uint32_t o_phi = off;  off += (uint32_t)ka_max * C::PHI_ATOM;
    const uint32_t o_x = off;    off += (uint32_t)nstage * STAGE_BYTES;
    const uint32_t o_recv = off; off += (uint32_t)NSLOT_P * S * C::PART * 4u;
    const uint32_t o_stg = off;  off += 2u * S * C::PART * 4u;     // two staging blocks
    const uint32_t o_hpre = off; off += (uint32_t)NSLOT_H * NT * 16u;
    const uint32_t o_ring = off; off += (uint32_t)RING * M * 4u;
    off = (off + 15u) & ~15u;
    const uint32_t o_bar = off;  off += B_COUNT * 8u;
    const uint32_t o_misc = off;
    float* recv = reinterpret_cast<float*>(sb + o_recv);
    float* stg = reinterpret_cast<float*>(sb + o_stg);
    float* hpre = reinterpret_cast<float*>(sb + o_hpre);
    float* ring = reinterpret_cast<float*>(sb + o_ring);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sb + o_misc);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sb + o_misc + 4);
    auto bar = [&](int i) -> uint32_t { return base + o_bar + 8u * (uint32_t)i; };
    const Waiter wait{abort_flag, wait_ns};
    const Waiter drain{abort_flag, wait_ns > kWaitNs ? wait_ns : kWaitNs};   // drains keep the full limit

    const int num_tiles = (T + NT - 1) / NT;
    const int cid = (int)cluster_idx(), ncl = (int)cluster_count();
    const int my_tiles = cid < num_tiles ? (num_tiles - cid + ncl - 1) / ncl : 0;

    // ---------------- set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; ++s) {
            mbar_init(bar(B_FULL + s), 1);
            mbar_init(bar(B_EMPTY + s), NMMA + 4);   // issuers' commits + 4 sum-of-squares warps
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(bar(B_ACCF + b), NMMA);
            mbar_init(bar(B_ACCE + b), 4);
        }
        for (int sl = 0; sl < NSLOT_P; ++sl) {
            mbar_init(bar(B_PFULL + sl), 1);
            mbar_init(bar(B_PEMPTY + sl), S);         // one remote arrive per owner
        }
        for (int sl = 0; sl < NSLOT_H; ++sl) {
            mbar_init(bar(B_HFULL + sl), 1);
            mbar_init(bar(B_HEMPTY + sl), S);         // one remote arrive per CTA's x_in warps
        }
        for (int i = 0; i < NMMA; ++i) mbar_init(bar(B_DRAIN + i), 1);
        for (int b = 0; b < 2; ++b) mbar_init(bar(B_STG_FREE + b), 1);   // warp 4: copies have read block b
        mbar_init(bar(B_STG_READY), 4);              // the 4 epilogue warps staged their rows
        for (int sl = 0; sl < NSLOT_H; ++sl) mbar_init(bar(B_XDONE + sl), NXW);   // x_in warps done
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(B_LG_FULL + b), 1);       // owner: a pass of logits is complete
            mbar_init(bar(B_LG_EMPTY + b), 1);      // Sinkhorn warp: the pass is consumed
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), (uint32_t)TMEM_COLS);

    // phi slice -> shared memory: atom al, row j < M = phi_hi column j, row M + j = phi_lo
    // column j, rows past 2M zero; 64 K values per row, 128-byte swizzle
    for (int idx = warp; idx < ka * 8; idx += NWARPS) {
        const int al = idx >> 3, c8 = idx & 7;
        const int64_t k0 = (int64_t)(a_lo + al) * 64 + c8 * 8;
        uint8_t* atom = sb + o_phi + (uint32_t)al * C::PHI_ATOM;
        if (lane < M) {
            float hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float v = __ldg(phi + (k0 + e) * M + lane);
                hi[e] = __bfloat162float(__float2bfloat16_rn(v));
                lo[e] = v - hi[e];
            }
            *reinterpret_cast<uint4*>(atom + sw128_off(lane, c8)) = Vec16<__nv_bfloat16>::pack(hi);
            *reinterpret_cast<uint4*>(atom + sw128_off(M + lane, c8)) = Vec16<__nv_bfloat16>::pack(lo);
        } else if (lane < M + (NB - 2 * M)) {
            *reinterpret_cast<uint4*>(atom + sw128_off(M + lane, c8)) = make_uint4(0, 0, 0, 0);
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int sl = 0; sl < NSLOT_P; ++sl) mbar_arrive_tx(bar(B_PFULL + sl), C::TX_PART);
        for (int sl = 0; sl < NSLOT_H; ++sl) mbar_arrive_tx(bar(B_HFULL + sl), C::TX_HPRE);
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---------------- roles
    if (warp == 0) {
        // TMA producer: stage g of the CTA holds atoms [al, al + na) of one tile
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.box[SA - 1]) : "memory");
            // stage g = (tile k = g / spt, atoms from al = (g % spt) * SA); the test hook stops
            // every CTA at the same tile
            const int spt = (ka + SA - 1) / SA;
            const int ntile = stop_tile >= 0 && stop_tile < my_tiles ? stop_tile : my_tiles;
            const int total = ntile * spt;
            // the box of stage g: tile origin and first atom
            auto stage_box = [&](int gg, int& t0, int& al, int& na) {
                const int k = gg / spt;
                al = (gg - k * spt) * SA;
                na = ka - al < SA ? ka - al : SA;
                t0 = (cid + k * ncl) * NT;
            };
            // L2 prefetch PF stages ahead: by the time a stage's load is issued its data is in
            // L2, so a slot of the ring turns over in an L2 round trip, not an HBM one
            for (int gg = 0; gg < PF && gg < total; ++gg) {
                int t0, al, na;
                stage_box(gg, t0, al, na);
                tma_prefetch_3d(&maps.box[na - 1], 0, t0, a_lo + al);
            }
            int g = 0;
            for (; g < total; ++g) {
                int t0, al, na;
                stage_box(g, t0, al, na);
                const int s = g % nstage, u = g / nstage;
                if (!wait(bar(B_EMPTY + s), (u & 1) ^ 1, E_EMPTY)) break;
                mbar_arrive_tx(bar(B_FULL + s), (uint32_t)(na * NT * 128));
                tma_load_3d(base + o_x + (uint32_t)s * STAGE_BYTES, &maps.box[na - 1], bar(B_FULL + s),
                            0, t0, a_lo + al);
                if (g + PF < total) {
                    int pt0, pal, pna;
                    stage_box(g + PF, pt0, pal, pna);
                    tma_prefetch_3d(&maps.box[pna - 1], 0, pt0, a_lo + pal);
                }
            }
            // drain: every issued copy has landed before the CTA can leave
            for (int j = g - 1; j >= 0 && j >= g - nstage; --j)
                drain(bar(B_FULL + j % nstage), (j / nstage) & 1, E_DRAIN, false);
        }
        __syncwarp();
    } else if (warp == 2 || warp == 3) {
        // MMA issuers: issuer i takes atoms i, i + NMMA, ... of every stage, into accumulator i
        const int i = warp - 2;
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_m64(NB);
            int g = 0, issued = 0;
            bool stop = false;
            for (int k = 0; k < my_tiles && !stop; ++k) {
                const int b = k % NACC, ub = k / NACC;
                if (!wait(bar(B_ACCE + b), (ub & 1) ^ 1, E_ACCE)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)((b * NMMA + i) * ACC_STRIDE);
                uint32_t accumulate = 0;
                for (int al = 0; al < ka; al += SA, ++g) {
                    const int s = g % nstage, u = g / nstage;
                    if (!wait(bar(B_FULL + s), u & 1, E_FULL_MMA)) { stop = true; break; }
                    tc_fence_after();
                    for (int j = i; j < SA && al + j < ka; j += NMMA) {
                        const uint64_t ad = sw128_desc(base + o_x + (uint32_t)s * STAGE_BYTES + (uint32_t)j * (NT * 128));
                        const uint64_t bd = sw128_desc(base + o_phi + (uint32_t)(al + j) * C::PHI_ATOM);
                        mma_bf16(d_tmem, ad, bd, IDESC, accumulate);
                        mma_bf16(d_tmem, ad + 2, bd + 2, IDESC, 1);
                        mma_bf16(d_tmem, ad + 4, bd + 4, IDESC, 1);
                        mma_bf16(d_tmem, ad + 6, bd + 6, IDESC, 1);
                        accumulate = 1;
                        issued = 1;
                    }
                    mma_commit(bar(B_EMPTY + s));
                }
                if (stop) break;
                mma_commit(bar(B_ACCF + b));
            }
            if (issued) {   // every MMA of this issuer completes before TMEM is released
                mma_commit(bar(B_DRAIN + i));
                drain(bar(B_DRAIN + i), 0, E_DRAIN, false);
            }
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // sums of squares (thread = token 16q + lane % 16, half lane / 16 of each 128-byte
        // row), then the accumulator epilogue (lanes < 16: TMEM lane 32q + lane = token 16q + lane)
        const int q = warp & 3;
        const int row = 16 * q + (lane & 15), half = lane >> 4;
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        int g = 0;
        for (int k = 0; k < my_tiles; ++k) {
            float2 sv[4];                         // eight independent FMA chains, in pairs
#pragma unroll
            for (int e = 0; e < 4; ++e) sv[e] = make_float2(0.f, 0.f);
            bool ok = true;
            for (int al = 0; al < ka; al += SA, ++g) {
                const int na = ka - al < SA ? ka - al : SA;
                const int s = g % nstage, u = g / nstage;
                if (!wait(bar(B_FULL + s), u & 1, E_FULL_SS)) { ok = false; break; }
                const uint8_t* xs = sb + o_x + (uint32_t)s * STAGE_BYTES + (uint32_t)row * 128;
#pragma unroll
                for (int a = 0; a < SA; ++a) {
                    if (a < na) {
                        uint4 w[4];
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            w[kk] = *reinterpret_cast<const uint4*>(xs + a * (NT * 128) + (((half * 4 + kk) ^ (row & 7)) << 4));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t ww[4] = {w[kk].x, w[kk].y, w[kk].z, w[kk].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = bf16x2_to_f32x2(ww[e]);
                                sv[e] = __ffma2_rn(f, f, sv[e]);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_EMPTY + s));
            }
            if (!ok) break;
            float ss = ((sv[0].x + sv[0].y) + (sv[1].x + sv[1].y)) + ((sv[2].x + sv[2].y) + (sv[3].x + sv[3].y));
            ss += __shfl_xor_sync(0xffffffffu, ss, 16);
            // accumulators of tile k: sum the issuers' partial projections
            const int b = k % NACC, ub = k / NACC;
            if (!wait(bar(B_ACCF + b), ub & 1, E_ACCF)) break;
            tc_fence_after();
            // one accumulator per round: all its columns in flight, then one wait
            constexpr int LW = NB % 16 == 0 ? 16 : 8;
            float acc[NB];
#pragma unroll
            for (int j = 0; j < NB; ++j) acc[j] = 0.f;
            for (int i = 0; i < nchain; ++i) {
                uint32_t r[NB];
#pragma unroll
                for (int c = 0; c < NB / LW; ++c)
                    tmem_ld_nowait<LW>(tq + (uint32_t)((b * NMMA + i) * ACC_STRIDE + c * LW), r + c * LW);
#pragma unroll
                for (int c8 = 0; c8 < NB / 8; ++c8) tmem_wait_regs8(r + c8 * 8);
#pragma unroll
                for (int j = 0; j < NB; ++j) acc[j] += __uint_as_float(r[j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_ACCE + b));
            // stage [h partial (hi + lo) | sum of squares] for the token's owner (lane % 16) in
            // block k % 2, once tile k-2's copies have read it
            const int sb2 = k & 1;
            float* stgk = stg + sb2 * S * C::PART;
            if (!wait(bar(B_STG_FREE + sb2), ((k >> 1) & 1) ^ 1, E_STG)) break;
            if (lane < 16) {
                float* dst = stgk + (lane * TPO + q) * W;
#pragma unroll
                for (int j = 0; j < M; ++j) dst[j] = acc[j] + acc[M + j];
                dst[M] = ss;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_STG_READY));
            if (q == 0) {
                // warp 4 ships the 16 owners' blocks, one bulk copy each
                if (!wait(bar(B_STG_READY), k & 1, E_STG)) break;
                if (lane < S) {
                    const int slot = k % NSLOT_P, us = k / NSLOT_P;
                    if (wait(bar(B_PEMPTY + slot), (us & 1) ^ 1, E_PEMPTY)) {
                        const uint32_t dst = base + o_recv + (uint32_t)((slot * S + (int)rank) * C::PART) * 4u;
                        bulk_to_peer(mapa(dst, (uint32_t)lane), smem_u32(stgk + lane * C::PART),
                                     (uint32_t)(C::PART * 4), mapa(bar(B_PFULL + slot), (uint32_t)lane));
                    }
                    bulk_wait_read_allbut1();     // tile k-1's copies have read their block
                }
                __syncwarp();
                if (lane == 0 && k > 0) mbar_arrive(bar(B_STG_FREE + (sb2 ^ 1)));
            }
        }
        if (q == 0 && lane < S) bulk_wait_all();
    } else if (warp == 1) {
        // owner: local tokens rank, rank + 16, rank + 32, rank + 48 of every tile
        const float invK = 1.0f / (float)(N * d);
        float bias = 0.f, alpha = 0.f;            // lane j's logit bias and gate scalar
        if (lane < N) { bias = __ldg(b_pre + lane); alpha = a_pre; }
        else if (lane < N + N * N) { bias = __ldg(b_res + (lane - N)); alpha = a_res; }
        else if (lane < M) { bias = __ldg(b_post + (lane - N - N * N)); alpha = a_post; }
        for (int k = 0; k < my_tiles; ++k) {
            const int slot = k % NSLOT_P, us = k / NSLOT_P;
            if (!wait.template operator()<true>(bar(B_PFULL + slot), us & 1, E_PFULL)) break;
            const float* rb = recv + slot * S * C::PART;
            float v[TPO];
#pragma unroll
            for (int t = 0; t < TPO; ++t) {
                float a = 0.f;
                if (lane < W) {
#pragma unroll
                    for (int src = 0; src < S; ++src) a += rb[src * C::PART + t * W + lane];
                }
                v[t] = a;
            }
            __syncwarp();
            // release the receive slot: arm its next phase, then tell the 16 senders
            if (lane == 0) mbar_arrive_tx(bar(B_PFULL + slot), C::TX_PART);
            __syncwarp();
            if (lane < S) mbar_arrive_remote(mapa(bar(B_PEMPTY + slot), (uint32_t)lane));
            const int t0 = (cid + k * ncl) * NT;
            float hp[TPO], zt[TPO];
#pragma unroll
            for (int t = 0; t < TPO; ++t) {
                const float ssum = __shfl_sync(0xffffffffu, v[t], M);
                const float inv_r = 1.0f / sqrtf(ssum * invK + eps);
                const float hn = v[t] * inv_r;
                const int64_t tok = (int64_t)t0 + t * S + (int)rank;
                if (h_out != nullptr && lane < M && tok < T) h_out[tok * M + lane] = hn;
                // mHC: logit z, gates and (Sinkhorn warp) Sinkhorn; HC: the coefficient itself
                const float z = hc ? bias + alpha * tanhf(hn) : alpha * hn + bias;
                const float pre = hc ? z : sigmoid_f32(z);
                hp[t] = lane < N ? pre : 0.f;
                zt[t] = lane < N ? pre : z;
            }
            // H_pre of the owner's tokens -> H_pre slot of every CTA of the cluster
            const int slh = k % NSLOT_H, uh = k / NSLOT_H;
            if (!wait(bar(B_HEMPTY + slh), (uh & 1) ^ 1, E_HEMPTY)) break;
#pragma unroll
            for (int t = 0; t < TPO; ++t) {
                float h4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) h4[i] = __shfl_sync(0xffffffffu, hp[t], i < N ? i : 31);
                if (lane < S) {
                    const uint32_t dst = smem_u32(hpre + (slh * NT + t * S + (int)rank) * 4);
                    st_async_v4(mapa(dst, (uint32_t)lane), h4[0], h4[1], h4[2], h4[3],
                                mapa(bar(B_HFULL + slh), (uint32_t)lane));
                }
            }
            // [H_pre | res logits | post logits] of the owner's tokens -> the Sinkhorn ring;
            // a pass is BATCH / TPO tiles
            const int kb = k % (BATCH / TPO), pb = k / (BATCH / TPO), b = pb & 1;
            if (kb == 0 && !wait(bar(B_LG_EMPTY + b), ((pb >> 1) & 1) ^ 1, E_LG_EMPTY)) break;
            if (lane < M) {
#pragma unroll
                for (int t = 0; t < TPO; ++t) ring[(b * BATCH + kb * TPO + t) * M + lane] = zt[t];
            }
            __syncwarp();
            if (lane == 0 && (kb == BATCH / TPO - 1 || k == my_tiles - 1)) mbar_arrive(bar(B_LG_FULL + b));
        }
    } else if (warp == SK_WARP) {
        // Sinkhorn-Knopp (H_res), H_post and the H store: one token per lane, BATCH tokens
        // (BATCH / TPO tiles of this owner) per pass
        const int npass = (my_tiles + BATCH / TPO - 1) / (BATCH / TPO);
        for (int pb = 0; pb < npass; ++pb) {
            const int b = pb & 1;
            if (!wait(bar(B_LG_FULL + b), (pb >> 1) & 1, E_LG_FULL)) break;
            const int k = pb * (BATCH / TPO) + lane / TPO, t = lane % TPO;
            if (k < my_tiles) {
                const float* L = ring + (b * BATCH + lane) * M;
                const int64_t tok = (int64_t)(cid + k * ncl) * NT + t * S + (int)rank;
                float out[M];
#pragma unroll
                for (int j = 0; j < M; ++j) out[j] = L[j];
                if (!hc) {
                    float Mx[N][N];
#pragma unroll
                    for (int i = 0; i < N; ++i)
#pragma unroll
                        for (int j = 0; j < N; ++j) Mx[i][j] = expf(out[N + i * N + j]);
                    sinkhorn_rounds<N>(Mx, t_max);
#pragma unroll
                    for (int i = 0; i < N; ++i)
#pragma unroll
                        for (int j = 0; j < N; ++j) out[N + i * N + j] = Mx[i][j];
#pragma unroll
                    for (int i = 0; i < N; ++i) out[N + N * N + i] = 2.0f * sigmoid_f32(out[N + N * N + i]);
                }
                if (tok < T) {
#pragma unroll
                    for (int j = 0; j < M; ++j) H[tok * M + j] = out[j];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_LG_EMPTY + b));
        }
    } else if (warp >= 8 && warp < 8 + NXW) {
        // x_in: this thread's tasks are xt, xt + NXT, ... of the tile's (token t, 8-channel
        // chunk c of this CTA's share) pairs, walked with increments; a tile's first round
        // of loads is issued before its H_pre arrives (the loads do not depend on it)
        constexpr int NXT = NXW * 32;
        const int xt = threadIdx.x - 8 * 32;
        const uint64_t pol = policy_evict_first();
        const int st = NXT / nch, sc = NXT % nch;
        const int t_first = xt / nch, c_first = xt % nch;
        const int xrow = N * d;                      // elements of X per token
        for (int k = 0; k < my_tiles; ++k) {
            const int slh = k % NSLOT_H, uh = k / NSLOT_H;
            const int64_t t0 = (int64_t)(cid + k * ncl) * NT;
            const int nt = T - t0 < NT ? (int)(T - t0) : NT;          // tokens of this tile
            const __nv_bfloat16* xb = X + t0 * xrow + (int64_t)c_lo * 8;
            __nv_bfloat16* ob = x_in + t0 * d + (int64_t)c_lo * 8;
            int t = t_first, c = c_first;
            uint4 xv[XU][N];
            int tt[XU], cc[XU];
            auto load_round = [&]() {
#pragma unroll
                for (int u = 0; u < XU; ++u) {
                    tt[u] = t;
                    cc[u] = c;
                    if (t < nt) {
                        const __nv_bfloat16* src = xb + (t * xrow + c * 8);
#pragma unroll
                        for (int i = 0; i < N; ++i) xv[u][i] = ld_last_use_v4(src + i * d, pol);
                    }
                    t += st;
                    c += sc;
                    if (c >= nch) { c -= nch; ++t; }
                }
            };
            load_round();
            if (!wait.template operator()<true>(bar(B_HFULL + slh), uh & 1, E_HFULL)) break;
            const float* hs = hpre + slh * NT * 4;
            while (true) {
#pragma unroll
                for (int u = 0; u < XU; ++u) {
                    if (tt[u] < nt) {
                        const float4 h4 = *reinterpret_cast<const float4*>(hs + tt[u] * 4);
                        const float hv[4] = {h4.x, h4.y, h4.z, h4.w};
                        float2 acc[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[e] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int i = 0; i < N; ++i) {
                            const float2 h2 = make_float2(hv[i], hv[i]);
                            const uint32_t ww[4] = {xv[u][i].x, xv[u][i].y, xv[u][i].z, xv[u][i].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) acc[e] = __ffma2_rn(h2, bf16x2_to_f32x2(ww[e]), acc[e]);
                        }
                        st_v4(ob + (tt[u] * d + cc[u] * 8),
                              make_uint4(pack_bf16x2(acc[0].x, acc[0].y), pack_bf16x2(acc[1].x, acc[1].y),
                                         pack_bf16x2(acc[2].x, acc[2].y), pack_bf16x2(acc[3].x, acc[3].y)));
                    }
                }
                if (t >= nt) break;
                load_round();
            }
            // once every x_in warp is done with the slot, warp 8 arms its next phase and
            // releases it to the 16 owners
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_XDONE + slh));
            if (warp == 8) {
                if (!wait(bar(B_XDONE + slh), uh & 1, E_XDONE)) break;
                if (lane == 0) mbar_arrive_tx(bar(B_HFULL + slh), C::TX_HPRE);
                __syncwarp();
                if (lane < S) mbar_arrive_remote(mapa(bar(B_HEMPTY + slh), (uint32_t)lane));
            }
        }
    }

    // ---------------- tear-down: no peer touches this CTA's shared memory after this
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
struct Plan {
    bool ok = false;
    int nstage = 0, smem = 0, max_clusters = 0, ka_max = 0;
};

template <int N>
int smem_bytes(int ka_max, int nstage) {
    using C = Cfg<N>;
    int off = ka_max * C::PHI_ATOM + nstage * STAGE_BYTES + NSLOT_P * S * C::PART * 4 + 2 * S * C::PART * 4 +
              NSLOT_H * NT * 16 + RING * C::M * 4;
    off = (off + 15) & ~15;
    off += B_COUNT * 8 + 16;
    off += 1024;         // alignment slack of the dynamic shared-memory base
    return off;
}

template <int N>
Plan make_plan(int d) {
    Plan p;
    DeviceInfo di;
    if (device_info(&di) != cudaSuccess || di.cc_major != 10 || di.cc_minor != 0) return p;
    const int ka_total = N * d / 64;
    const int ka_max = (ka_total + S - 1) / S;
    int ns = MAXST;
    while (ns >= 2 && smem_bytes<N>(ka_max, ns) > di.max_smem_optin) --ns;
    if (ns < 2) return p;
    const int smem = smem_bytes<N>(ka_max, ns);
    auto kern = pre_tc_kernel<N>;
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
    p.ka_max = ka_max;
    return p;
}

// plans cached per (device, n, d)
Plan get_plan(int n, int d) {
    struct Key { int dev, n, d; };
    constexpr int kCache = 256;
    static std::mutex mu;
    static Key keys[kCache];
    static Plan plans[kCache];
    static int used = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || n < 1 || n > 4) {
        cudaGetLastError();
        return Plan{};
    }
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i)
        if (keys[i].dev == dev && keys[i].n == n && keys[i].d == d) return plans[i];
    Plan p;
    switch (n) {
        case 1: p = make_plan<1>(d); break;
        case 2: p = make_plan<2>(d); break;
        case 3: p = make_plan<3>(d); break;
        case 4: p = make_plan<4>(d); break;
    }
    if (used < kCache) {
        keys[used] = Key{dev, n, d};
        plans[used] = p;
        ++used;
    }
    return p;
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

// test hook of the failure path (see mhc_debug_pre_stop_after): tiles per cluster after
// which the producers stop, and the wait limit
std::atomic<int> g_stop_tile{-1};
std::atomic<unsigned long long> g_wait_ns{kWaitNs};

template <int N>
cudaError_t launch_n(const PreArgs& a, const Plan& p) {
    // X viewed as 3-D: (element within a 64-channel atom: 64, token: T, atom: n d / 64);
    // box j: (64, NT, j + 1) -- j + 1 atoms of NT tokens, stored atom-major
    Maps maps;
    const int ka_total = N * a.d / 64;
    const cuuint64_t dims[3] = {64, (cuuint64_t)a.T, (cuuint64_t)ka_total};
    const cuuint64_t strides[2] = {(cuuint64_t)N * a.d * 2, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    for (int j = 0; j < SA; ++j) {
        const cuuint32_t box[3] = {64, (cuuint32_t)NT, (cuuint32_t)(j + 1)};
        CUresult r = enc(&maps.box[j], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.X), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
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
    return cudaLaunchKernelEx(&cfg, pre_tc_kernel<N>, maps, static_cast<const __nv_bfloat16*>(a.X), a.phi,
                              a.b_pre, a.b_post, a.b_res, a.a_pre, a.a_post, a.a_res, (int)a.T, a.d, a.eps,
                              a.t_max, static_cast<__nv_bfloat16*>(a.x_in), a.H, a.h_out, ka_total, p.ka_max,
                              p.nstage, g_stop_tile.load(), g_wait_ns.load(), a.hc ? 1 : 0);
}

}  // namespace tc

bool pre_tc_shape_ok(int64_t T, int n, int d, DType dt) {
    return dt == BF16 && n >= 1 && n <= 4 && d % 64 == 0 && (int64_t)n * d >= 64 * tc::S &&
           T >= 1 && T < ((int64_t)1 << 31) - tc::NT;
}

bool pre_tc_device_ok(int n, int d) {
    if (n < 1 || n > 4 || d % 64 != 0 || n * d < 64 * tc::S) return false;
    return tc::get_plan(n, d).ok;
}

cudaError_t launch_pre_tc(const PreArgs& a) {
    const tc::Plan p = tc::get_plan(a.n, a.d);
    if (!p.ok) return cudaErrorNotSupported;
    switch (a.n) {
        case 1: return tc::launch_n<1>(a, p);
        case 2: return tc::launch_n<2>(a, p);
        case 3: return tc::launch_n<3>(a, p);
        case 4: return tc::launch_n<4>(a, p);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t pre_tc_status(unsigned* out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_pre_tc_status, sizeof(unsigned));
    if (e != cudaSuccess) return e;
    if (clear && *out) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_pre_tc_status, &zero, sizeof(unsigned));
    }
    return e;
}

void pre_tc_set_stop(int stop_tile, unsigned long long wait_ns) {
    tc::g_stop_tile.store(stop_tile);
    tc::g_wait_ns.store(wait_ns);
}

}  // namespace mhc
