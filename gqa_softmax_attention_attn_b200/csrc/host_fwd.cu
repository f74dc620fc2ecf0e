// host_fwd.cu -- the bf16 prefill forward with its inputs and outputs in host
// memory, the transfers overlapped with the computation.
//
// What it computes is attn_sink_fwd's forward ("GPT-OSS on day 0", section
// "Sink Attention").  What makes the overlap possible is causality: the rows of
// query positions [p0, p1) see keys below p1 + (Lk - Lq) only, so a chunk of
// positions can run as soon as its q rows and the keys up to its last position
// are on the device, while the next chunk's rows are still on their way in
// and the previous chunk's output is on its way out.
//
// Design: three streams per call -- host-to-device copies on one of the
// library's own streams, the forward kernels on the caller's stream, and
// device-to-host copies on a second stream of the library's own -- joined by
// one event per chunk in each direction.  The first copy waits for the work
// already on the caller's stream (the workspace may be in use there), and the
// caller's stream waits for the last copy, so the call is ordered on that
// stream as a whole.  Chunks start at multiples of 128 positions, a multiple
// of the forward kernels' item height (128 rows / the query heads packed per
// item), so the items, their tiles and every row's arithmetic are those of a
// single launch over all positions.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "kernels.h"

namespace attn_sink {
namespace {

constexpr int kMaxDevs = 64;

// The copy streams and events of a device, made on first use and kept; a
// call holds the device's lock while it enqueues its work.
struct HostPipe {
    std::mutex mu;
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, end = nullptr;
    cudaEvent_t in[kFwdHostMaxChunks], out[kFwdHostMaxChunks];
};
HostPipe g_pipe[kMaxDevs];

cudaError_t pipe_init(HostPipe &hp)
{
    cudaError_t e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.end, cudaEventDisableTiming);
    for (int c = 0; c < kFwdHostMaxChunks && e == cudaSuccess; ++c) {
        e = cudaEventCreateWithFlags(&hp.in[c], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.out[c], cudaEventDisableTiming);
    }
    return e;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Chunk c of the Lq positions spans [bnd[c], bnd[c + 1]); returns the number of
// chunks (at most n).  The first chunk's copy-in and the last chunk's kernel
// and copy-out overlap nothing, so with three or more chunks those two get
// weight 1 and the others weight 2; every end but the last is rounded to a
// whole 128-position block.  (Four chunks of a B1 L4096 dense layer: 1.21 ms
// against 1.29-1.30 ms for equal chunks.)
int chunk_bounds(int Lq, int n, int *bnd)
{
    const long long wsum = n <= 2 ? n : 2 * (long long)n - 2;
    long long cum = 0;
    int nc = 0;
    bnd[0] = 0;
    for (int c = 0; c < n; ++c) {
        cum += (n <= 2 || c == 0 || c == n - 1) ? 1 : 2;
        int e = (int)((Lq * cum + wsum / 2) / wsum);
        e = c == n - 1 ? Lq : (e + 64) / 128 * 128;
        if (e > Lq) e = Lq;
        if (e > bnd[nc]) bnd[++nc] = e;
    }
    return nc;
}

}  // namespace

size_t fwd_host_workspace_bytes(const AttnShape &s)
{
    const size_t qb = (size_t)s.B * s.Lq * s.Hq * s.D * 2, kvb = (size_t)s.B * s.Lk * s.Hkv * s.D * 2;
    return 2 * align256(qb) + 2 * align256(kvb) + align256((size_t)s.B * s.Hq * s.Lq * 4) + align256((size_t)s.Hq * 4);
}

cudaError_t run_fwd_host(const void *q_h, const void *k_h, const void *v_h, const float *sinks_h, void *out_h,
                         float *lse_h, const AttnShape &s, int n_chunks, void *workspace, cudaStream_t st)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevs) return cudaErrorInvalidDevice;
    HostPipe &hp = g_pipe[dev];
    std::lock_guard<std::mutex> lock(hp.mu);
    if (!hp.ready) {
        e = pipe_init(hp);
        if (e != cudaSuccess) return e;
        hp.ready = true;
    }

    // workspace: q | k | v | out | lse ([B, Hq, Lq], as on the host) | sinks
    const size_t row_q = (size_t)s.Hq * s.D * 2, row_kv = (size_t)s.Hkv * s.D * 2;  // bytes per position
    uint8_t *w = static_cast<uint8_t *>(workspace);
    uint8_t *q_d = w;
    w += align256((size_t)s.B * s.Lq * row_q);
    uint8_t *k_d = w;
    w += align256((size_t)s.B * s.Lk * row_kv);
    uint8_t *v_d = w;
    w += align256((size_t)s.B * s.Lk * row_kv);
    uint8_t *out_d = w;
    w += align256((size_t)s.B * s.Lq * row_q);
    float *lse_d = reinterpret_cast<float *>(w);
    w += align256((size_t)s.B * s.Hq * s.Lq * 4);
    float *sinks_d = reinterpret_cast<float *>(w);

    const uint8_t *qh = static_cast<const uint8_t *>(q_h), *kh = static_cast<const uint8_t *>(k_h),
                  *vh = static_cast<const uint8_t *>(v_h);
    uint8_t *oh = static_cast<uint8_t *>(out_h);
    const int off = s.Lk - s.Lq;  // >= 0
    int bnd[kFwdHostMaxChunks + 1];
    const int nc = chunk_bounds(s.Lq, n_chunks, bnd);  // whole items per chunk

#define ATTN_SINK_CK(x)                  \
    do {                                 \
        e = (x);                         \
        if (e != cudaSuccess) return e;  \
    } while (0)
    ATTN_SINK_CK(cudaEventRecord(hp.start, st));
    ATTN_SINK_CK(cudaStreamWaitEvent(hp.h2d, hp.start, 0));
    ATTN_SINK_CK(cudaStreamWaitEvent(hp.d2h, hp.start, 0));
    ATTN_SINK_CK(cudaMemcpyAsync(sinks_d, sinks_h, (size_t)s.Hq * 4, cudaMemcpyHostToDevice, hp.h2d));
    int kv_done = 0;  // key rows already sent (the same for every batch element)
    for (int c = 0; c < nc; ++c) {
        const int p0 = bnd[c], p1 = bnd[c + 1];
        const int kneed = p1 + off;  // keys the chunk's rows can see
        const size_t nq = (size_t)(p1 - p0) * row_q;
        // in: the chunk's q rows and the keys it adds
        for (int b = 0; b < s.B; ++b) {
            const size_t qo = ((size_t)b * s.Lq + p0) * row_q;
            ATTN_SINK_CK(cudaMemcpyAsync(q_d + qo, qh + qo, nq, cudaMemcpyHostToDevice, hp.h2d));
            if (kneed > kv_done) {
                const size_t ko = ((size_t)b * s.Lk + kv_done) * row_kv, nk = (size_t)(kneed - kv_done) * row_kv;
                ATTN_SINK_CK(cudaMemcpyAsync(k_d + ko, kh + ko, nk, cudaMemcpyHostToDevice, hp.h2d));
                ATTN_SINK_CK(cudaMemcpyAsync(v_d + ko, vh + ko, nk, cudaMemcpyHostToDevice, hp.h2d));
            }
        }
        if (kneed > kv_done) kv_done = kneed;
        ATTN_SINK_CK(cudaEventRecord(hp.in[c], hp.h2d));
        // the chunk's rows: positions [p0, p1) as the last p1 - p0 queries of a
        // sequence of kneed keys, one launch per batch element; lse goes to
        // columns [p0, p1) of the batch element's [Hq, Lq]
        ATTN_SINK_CK(cudaStreamWaitEvent(st, hp.in[c], 0));
        for (int b = 0; b < s.B; ++b) {
            const size_t qo = ((size_t)b * s.Lq + p0) * row_q, ko = (size_t)b * s.Lk * row_kv;
            AttnShape cs{1, p1 - p0, kneed, s.Hq, s.Hkv, s.D, s.window, s.scale};
            cs.lse_hs = s.Lq;
            ATTN_SINK_CK(launch_fwd_tc(q_d + qo, k_d + ko, v_d + ko, sinks_d, out_d + qo,
                                       lse_d + (size_t)b * s.Hq * s.Lq + p0, cs, st));
        }
        ATTN_SINK_CK(cudaEventRecord(hp.out[c], st));
        // out: the chunk's output rows (lse, a few bytes per row, goes back
        // once at the end: copied per chunk, its Hq short rows cost more than
        // they carry)
        ATTN_SINK_CK(cudaStreamWaitEvent(hp.d2h, hp.out[c], 0));
        for (int b = 0; b < s.B; ++b) {
            const size_t qo = ((size_t)b * s.Lq + p0) * row_q;
            ATTN_SINK_CK(cudaMemcpyAsync(oh + qo, out_d + qo, nq, cudaMemcpyDeviceToHost, hp.d2h));
        }
    }
    ATTN_SINK_CK(cudaMemcpyAsync(lse_h, lse_d, (size_t)s.B * s.Hq * s.Lq * 4, cudaMemcpyDeviceToHost, hp.d2h));
    ATTN_SINK_CK(cudaEventRecord(hp.end, hp.d2h));
    ATTN_SINK_CK(cudaStreamWaitEvent(st, hp.end, 0));
#undef ATTN_SINK_CK
    return cudaSuccess;
}

}  // namespace attn_sink
