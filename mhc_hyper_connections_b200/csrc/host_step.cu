// host_step.cu -- mhc_forward_host: the pre and post stages (slavadubrov.com Eq. 3; the
// "DeepSeek-V4/mhc" page's pre kernel and post-res fused kernel) over activations that live in
// host memory.
//
// The tokens go through in chunks. Each chunk's inputs are copied into one of three device
// buffer sets, the two stages run on it on the caller's stream, and its outputs are copied
// back. The copy-in of chunk c + 1, the kernels of chunk c and the copy-out of chunk c - 1 run
// at the same time: the copies in and out use two streams of their own, so the PCIe link
// carries both directions at once. A chunk is a contiguous run of tokens, and every output of
// a token depends on that token alone. So the results are those of mhc_pre and mhc_post called
// on each chunk, whatever the chunk size.
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "launch.cuh"
#include "mhc.h"

namespace mhc {
mhc_status report_cuda_error(cudaError_t e, const char* where);
}

namespace {

constexpr int kSets = 3;          // device buffer sets in rotation
constexpr int kMaxDev = 64;

// Per-device copy streams and the events that order the three streams. They are created on
// the first call on a device and live as long as the process; calls on one device are
// serialised while they enqueue their work.
struct HostCtx {
    bool ready = false;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t in[kSets] = {}, comp[kSets] = {}, out[kSets] = {};
    std::mutex enqueue;
};
HostCtx g_ctx[kMaxDev];
std::mutex g_ctx_mu;

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// Byte offsets of one buffer set for chunks of ct tokens.
struct SetLayout {
    size_t X, F, xin, H, Y, total;
};

SetLayout set_layout(int64_t ct, int n, int d, size_t es) {
    const size_t m = (size_t)n * n + 2 * (size_t)n;
    SetLayout L;
    size_t off = 0;
    L.X = off;   off += round256((size_t)ct * n * d * es);
    L.F = off;   off += round256((size_t)ct * d * es);
    L.xin = off; off += round256((size_t)ct * d * es);
    L.H = off;   off += round256((size_t)ct * m * 4);
    L.Y = off;   off += round256((size_t)ct * n * d * es);
    L.total = off;
    return L;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (na == 0 || nb == 0) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Shape limits of mhc_pre, plus a chunk small enough that a buffer set stays under 2^40 bytes
// (a set holds at most 8 n d + 8 d + 320 bytes per token: X and X_out, F_out and x_in, H).
mhc_status check_args(int64_t T, int n, int d, int t_max, mhc_dtype dt, int64_t chunk_tokens) {
    if (dt != MHC_F32 && dt != MHC_BF16) return MHC_ERR_DTYPE;
    if (n < 1 || n > 8 || d < 1 || T < 0 || t_max < 0 || t_max > 1000) return MHC_ERR_SHAPE;
    const int64_t row = (int64_t)n * d;
    if (row > (int64_t)1 << 30) return MHC_ERR_SHAPE;
    if (T > (((int64_t)1 << 62) / (row * 8))) return MHC_ERR_SHAPE;
    const int64_t per_token = 8 * row + 8 * (int64_t)d + 320;
    if (chunk_tokens < 1 || chunk_tokens > ((int64_t)1 << 40) / per_token) return MHC_ERR_SHAPE;
    return MHC_OK;
}

mhc_status get_ctx(HostCtx** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return mhc::report_cuda_error(e, "mhc_forward_host");
    if (dev < 0 || dev >= kMaxDev) return mhc::report_cuda_error(cudaErrorInvalidDevice, "mhc_forward_host");
    std::lock_guard<std::mutex> lk(g_ctx_mu);
    HostCtx& c = g_ctx[dev];
    if (!c.ready) {
        e = cudaStreamCreateWithFlags(&c.s_in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c.s_out, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.start, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.done, cudaEventDisableTiming);
        for (int b = 0; b < kSets && e == cudaSuccess; ++b) {
            e = cudaEventCreateWithFlags(&c.in[b], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.comp[b], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.out[b], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) return mhc::report_cuda_error(e, "mhc_forward_host (stream / event set-up)");
        c.ready = true;
    }
    *out = &c;
    return MHC_OK;
}

}  // namespace

extern "C" {

size_t mhc_forward_host_workspace_bytes(int64_t chunk_tokens, int n, int d, mhc_dtype dt) {
    if (check_args(0, n, d, 0, dt, chunk_tokens) != MHC_OK) return 0;
    const size_t es = dt == MHC_BF16 ? 2 : 4;
    return (size_t)kSets * set_layout(chunk_tokens, n, d, es).total;
}

mhc_status mhc_forward_host(const void* X_h, const void* F_out_h, const float* phi,
                            const float* b_pre, const float* b_post, const float* b_res,
                            float alpha_pre, float alpha_post, float alpha_res, int64_t T, int n,
                            int d, float eps, int t_max, mhc_dtype dt, void* x_in_h, float* H_h,
                            void* X_out_h, int64_t chunk_tokens, void* workspace,
                            size_t workspace_bytes, mhc_stream_t stream) {
    mhc_status st = check_args(T, n, d, t_max, dt, chunk_tokens);
    if (st != MHC_OK) return st;
    if (T == 0) return MHC_OK;
    if (!X_h || !F_out_h || !phi || !b_pre || !b_post || !b_res || !x_in_h || !H_h || !X_out_h || !workspace)
        return MHC_ERR_NULL;
    const size_t es = dt == MHC_BF16 ? 2 : 4;
    const int m = n * n + 2 * n;
    if (!aligned(X_h, es) || !aligned(F_out_h, es) || !aligned(x_in_h, es) || !aligned(X_out_h, es) ||
        !aligned(H_h, 4) || !aligned(phi, 4) || !aligned(b_pre, 4) || !aligned(b_post, 4) ||
        !aligned(b_res, 4) || !aligned(workspace, 256))
        return MHC_ERR_ALIGN;
    const int64_t ct = chunk_tokens < T ? chunk_tokens : T;
    const SetLayout L = set_layout(ct, n, d, es);
    const size_t need = (size_t)kSets * L.total;
    if (workspace_bytes < need) return MHC_ERR_WORKSPACE;
    // host arrays: outputs overlap no input and no other output
    const size_t nX = (size_t)T * n * d * es, nD = (size_t)T * d * es, nH = (size_t)T * m * 4;
    const void* hin[2] = {X_h, F_out_h};
    const size_t nhin[2] = {nX, nD};
    void* hout[3] = {x_in_h, H_h, X_out_h};
    const size_t nhout[3] = {nD, nH, nX};
    for (int o = 0; o < 3; ++o) {
        for (int i = 0; i < 2; ++i)
            if (overlaps(hout[o], nhout[o], hin[i], nhin[i])) return MHC_ERR_ALIAS;
        for (int p = o + 1; p < 3; ++p)
            if (overlaps(hout[o], nhout[o], hout[p], nhout[p])) return MHC_ERR_ALIAS;
    }
    // the device workspace is written: it may not hold the parameters
    const void* par[4] = {phi, b_pre, b_post, b_res};
    const size_t npar[4] = {(size_t)n * d * m * 4, (size_t)n * 4, (size_t)n * 4, (size_t)n * n * 4};
    for (int i = 0; i < 4; ++i)
        if (overlaps(workspace, need, par[i], npar[i])) return MHC_ERR_ALIAS;

    HostCtx* c = nullptr;
    if ((st = get_ctx(&c)) != MHC_OK) return st;
    std::lock_guard<std::mutex> lk(c->enqueue);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto fail = [&](cudaError_t e) { return mhc::report_cuda_error(e, "mhc_forward_host"); };
    cudaError_t e = cudaEventRecord(c->start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c->s_in, c->start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c->s_out, c->start, 0);
    if (e != cudaSuccess) return fail(e);

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int64_t nchunks = (T + ct - 1) / ct;
    for (int64_t ci = 0; ci < nchunks; ++ci) {
        const int b = (int)(ci % kSets);
        const int64_t t0 = ci * ct, tc = T - t0 < ct ? T - t0 : ct;
        uint8_t* set = ws + (size_t)b * L.total;
        void* Xd = set + L.X;
        void* Fd = set + L.F;
        void* xd = set + L.xin;
        float* Hd = reinterpret_cast<float*>(set + L.H);
        void* Yd = set + L.Y;
        const size_t bX = (size_t)tc * n * d * es, bD = (size_t)tc * d * es, bH = (size_t)tc * m * 4;
        // copy in, once the set's previous chunk has been copied out
        if (ci >= kSets) e = cudaStreamWaitEvent(c->s_in, c->out[b], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(Xd, static_cast<const uint8_t*>(X_h) + (size_t)t0 * n * d * es, bX,
                                cudaMemcpyHostToDevice, c->s_in);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(Fd, static_cast<const uint8_t*>(F_out_h) + (size_t)t0 * d * es, bD,
                                cudaMemcpyHostToDevice, c->s_in);
        if (e == cudaSuccess) e = cudaEventRecord(c->in[b], c->s_in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, c->in[b], 0);
        if (e != cudaSuccess) return fail(e);
        // the two stages on the caller's stream
        st = mhc_pre(Xd, phi, b_pre, b_post, b_res, alpha_pre, alpha_post, alpha_res, tc, n, d, eps,
                     t_max, dt, xd, Hd, stream);
        if (st != MHC_OK) return st;
        st = mhc_post(Xd, Fd, Hd, tc, n, d, dt, Yd, stream);
        if (st != MHC_OK) return st;
        e = cudaEventRecord(c->comp[b], s);
        // copy out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(c->s_out, c->comp[b], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<uint8_t*>(x_in_h) + (size_t)t0 * d * es, xd, bD,
                                cudaMemcpyDeviceToHost, c->s_out);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(H_h) + (size_t)t0 * m * 4, Hd, bH,
                                cudaMemcpyDeviceToHost, c->s_out);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<uint8_t*>(X_out_h) + (size_t)t0 * n * d * es, Yd, bX,
                                cudaMemcpyDeviceToHost, c->s_out);
        if (e == cudaSuccess) e = cudaEventRecord(c->out[b], c->s_out);
        if (e != cudaSuccess) return fail(e);
    }
    // the caller's stream resumes once every copy out has landed
    e = cudaEventRecord(c->done, c->s_out);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, c->done, 0);
    if (e != cudaSuccess) return fail(e);
    return MHC_OK;
}

}  // extern "C"
