// simt_kernels.cu -- the exact CUDA-core path: prefill forward, backward and
// split-KV decode for fp32 (and, as a cross-check, bf16) inputs, plus the
// split combine that folds the sink into the final log-sum-exp exactly once
// ("GPT-OSS on day 0", section "Sink Attention").  Every score, exponential
// and accumulation is fp32 with accurate expf/exp2f, so fp32 inputs meet a
// 1e-5 max-abs bound.
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

constexpr int kD = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_max(float x)
{
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x)
{
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ bool visible(long j, long p, int window, int Lk)
{
    return j <= p && j < Lk && (window <= 0 || j > p - window);
}

// ------------------------------------------------------------------ forward
// CTA = 16 query rows of one head (4 warps x 4 rows); keys in tiles of 32,
// lane = key for the scores, lane = (d, d + 32) for the output.
template <typename T>
__global__ void __launch_bounds__(128) fwd_simt_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                       const T *__restrict__ v, const float *__restrict__ sinks,
                                                       T *__restrict__ out, float *__restrict__ lse, AttnShape s)
{
    __shared__ float qs[16][kD];
    __shared__ float ks[32][kD + 1];
    __shared__ float vs[32][kD];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i0 = blockIdx.x * 16, h = blockIdx.y, b = blockIdx.z;
    const int G = s.Hq / s.Hkv, g = h / G;
    const long off = (long)s.Lk - s.Lq;
    const size_t qrow = (size_t)s.Hq * kD, krow = (size_t)s.Hkv * kD;

    for (int e = tid; e < 16 * kD; e += 128) {
        const int r = e / kD, d = e % kD, i = i0 + r;
        qs[r][d] = i < s.Lq ? to_f(q[((size_t)b * s.Lq + i) * qrow + (size_t)h * kD + d]) : 0.f;
    }
    const int ilast = min(i0 + 15, s.Lq - 1);
    const long pmin = i0 + off, pmax = ilast + off;
    long lo = s.window > 0 ? max(0L, pmin - s.window + 1) : 0L;
    long hi = min((long)s.Lk, pmax + 1);  // exclusive

    const float sink = sinks[h];
    float m[4], l[4], o0[4], o1[4];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        m[rr] = sink;
        l[rr] = (sink == -INFINITY) ? 0.f : 1.f;
        o0[rr] = 0.f;
        o1[rr] = 0.f;
    }
    for (long j0 = (lo / 32) * 32; j0 < hi; j0 += 32) {
        __syncthreads();
        for (int e = tid; e < 32 * kD; e += 128) {
            const int r = e / kD, d = e % kD;
            const long j = j0 + r;
            const bool in = j < s.Lk;
            const size_t idx = ((size_t)b * s.Lk + (in ? j : 0)) * krow + (size_t)g * kD + d;
            ks[r][d] = in ? to_f(k[idx]) : 0.f;
            vs[r][d] = in ? to_f(v[idx]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const int r = warp * 4 + rr, i = i0 + r;
            if (i >= s.Lq) continue;
            const long p = i + off, j = j0 + lane;
            float sc = 0.f;
#pragma unroll 16
            for (int d = 0; d < kD; ++d) sc = fmaf(qs[r][d], ks[lane][d], sc);
            sc *= s.scale;
            const bool vis = visible(j, p, s.window, s.Lk);
            sc = vis ? sc : -INFINITY;
            const float mn = fmaxf(m[rr], warp_max(sc));
            if (mn == -INFINITY) continue;
            const float alpha = (m[rr] == -INFINITY) ? 0.f : expf(m[rr] - mn);
            const float pj = vis ? expf(sc - mn) : 0.f;
            l[rr] = l[rr] * alpha + warp_sum(pj);
            float a0 = o0[rr] * alpha, a1 = o1[rr] * alpha;
#pragma unroll 8
            for (int jj = 0; jj < 32; ++jj) {
                const float w = __shfl_sync(0xffffffffu, pj, jj);
                a0 = fmaf(w, vs[jj][lane], a0);
                a1 = fmaf(w, vs[jj][lane + 32], a1);
            }
            o0[rr] = a0;
            o1[rr] = a1;
            m[rr] = mn;
        }
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int r = warp * 4 + rr, i = i0 + r;
        if (i >= s.Lq) continue;
        const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
        T *orow = out + ((size_t)b * s.Lq + i) * qrow + (size_t)h * kD;
        orow[lane] = from_f<T>(o0[rr] * inv);
        orow[lane + 32] = from_f<T>(o1[rr] * inv);
        if (lane == 0)
            lse[((size_t)b * s.Hq + h) * s.Lq + i] = l[rr] > 0.f ? m[rr] + logf(l[rr]) : -INFINITY;
    }
}

// ------------------------------------------------------------------ backward
// (1) per row: D_i = <dO_i, O_i>, dsink term -exp(sink - lse_i) * D_i.
// HBM-bound (one read of O and dO): a row of 64 values is 128 or 256 bytes,
// read as 16-byte chunks by kTpr neighbouring threads (8 for bf16, 16 for
// fp32) whose partial dot products meet in a shuffle reduction; each thread
// takes kRowsPerThread rows with all their loads issued first, so enough bytes
// are in flight per SM to cover the memory latency.  When `zero` is given
// (the fp32 dQ accumulator of the tensor-core backward, rows in the same
// [B, Lq, Hq] order), the same threads clear its rows in this pass.
template <typename T>
struct PreRows {
    static constexpr int kElems = 16 / sizeof(T);  // values per 16-byte chunk
    static constexpr int kTpr = kD / kElems;       // threads per row
    static constexpr int kRowsPerThread = 2;  // with four CTAs per SM (measured best of 2/4/8 rows)
    static constexpr int kMinCtas = 4;
    static constexpr int kRowsPerCta = 256 / kTpr * kRowsPerThread;
};

__device__ __forceinline__ float dot16(const uint4 &a, const uint4 &b, float)
{
    const float *x = reinterpret_cast<const float *>(&a), *y = reinterpret_cast<const float *>(&b);
    return x[0] * y[0] + x[1] * y[1] + x[2] * y[2] + x[3] * y[3];
}
__device__ __forceinline__ float dot16(const uint4 &a, const uint4 &b, __nv_bfloat16)
{
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wa[j]));
        const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wb[j]));
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
    }
    return acc;
}

template <typename T>
__global__ void __launch_bounds__(256, PreRows<T>::kMinCtas) bwd_pre_kernel(const T *__restrict__ out, const T *__restrict__ dout,
                                                      const float *__restrict__ lse,
                                                      const float *__restrict__ sinks, float *__restrict__ Drow,
                                                      float *__restrict__ terms, float *__restrict__ zero,
                                                      AttnShape s)
{
    using R = PreRows<T>;
    // the backward's main kernel may start its set-up (it waits for this
    // grid before it reads D or adds into the accumulator)
    grid_dep_launch();
    const int sub = threadIdx.x % R::kTpr;  // chunk of the row
    const long nrows = (long)s.B * s.Lq * s.Hq;
    const long row0 = (long)blockIdx.x * R::kRowsPerCta + threadIdx.x / R::kTpr;
    constexpr int kStride = 256 / R::kTpr;  // rows between a thread's successive rows
    // every load of the thread's rows first (O, dO, and the row's lse and sink,
    // which all kTpr threads of the row read), so one memory latency covers them
    uint4 a[R::kRowsPerThread], b[R::kRowsPerThread];
    float Lr[R::kRowsPerThread], sk[R::kRowsPerThread];
    size_t li[R::kRowsPerThread], ti[R::kRowsPerThread];
#pragma unroll
    for (int u = 0; u < R::kRowsPerThread; ++u) {
        const long row = row0 + (long)u * kStride;
        if (row < nrows) {
            const size_t off = (size_t)row * kD + (size_t)sub * R::kElems;
            a[u] = *reinterpret_cast<const uint4 *>(out + off);
            b[u] = *reinterpret_cast<const uint4 *>(dout + off);
            int h, i, bb;  // row over [B, Lq, Hq]
            if (nrows <= 0xffffffffL) {  // 32-bit division where it suffices
                const uint32_t r32 = (uint32_t)row, bi = r32 / (uint32_t)s.Hq;
                h = (int)(r32 - bi * (uint32_t)s.Hq);
                bb = (int)(bi / (uint32_t)s.Lq);
                i = (int)(bi - (uint32_t)bb * (uint32_t)s.Lq);
            } else {
                h = (int)(row % s.Hq);
                const long bi = row / s.Hq;
                i = (int)(bi % s.Lq);
                bb = (int)(bi / s.Lq);
            }
            li[u] = ((size_t)bb * s.Hq + h) * s.Lq + i;
            ti[u] = (size_t)h * s.B * s.Lq + (size_t)bb * s.Lq + i;
            Lr[u] = lse[li[u]];
            sk[u] = sinks[h];
            if (zero) {
                constexpr int kF = kD / R::kTpr;  // fp32 values of the row per thread
                float4 *z = reinterpret_cast<float4 *>(zero + (size_t)row * kD + (size_t)sub * kF);
#pragma unroll
                for (int c = 0; c < kF / 4; ++c) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else {
            a[u] = b[u] = make_uint4(0u, 0u, 0u, 0u);
            Lr[u] = sk[u] = 0.f;
            li[u] = ti[u] = 0;
        }
    }
#pragma unroll
    for (int u = 0; u < R::kRowsPerThread; ++u) {
        float d = dot16(a[u], b[u], T{});
#pragma unroll
        for (int w = R::kTpr / 2; w > 0; w >>= 1) d += __shfl_xor_sync(0xffffffffu, d, w);
        const long row = row0 + (long)u * kStride;
        if (sub == 0 && row < nrows) {
            Drow[li[u]] = d;
            const float ps = (Lr[u] == -INFINITY) ? 0.f : expf(sk[u] - Lr[u]);
            terms[ti[u]] = -ps * d;
        }
    }
}

// (2) dq: CTA = 16 rows of one head, keys in tiles of 32.
template <typename T>
__global__ void __launch_bounds__(128) bwd_dq_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                     const T *__restrict__ v, const T *__restrict__ dout,
                                                     const float *__restrict__ lse, const float *__restrict__ Drow,
                                                     T *__restrict__ dq, AttnShape s)
{
    __shared__ float qs[16][kD], dos[16][kD];
    __shared__ float ks[32][kD + 1], vs[32][kD + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i0 = blockIdx.x * 16, h = blockIdx.y, b = blockIdx.z;
    const int G = s.Hq / s.Hkv, g = h / G;
    const long off = (long)s.Lk - s.Lq;
    const size_t qrow = (size_t)s.Hq * kD, krow = (size_t)s.Hkv * kD;
    for (int e = tid; e < 16 * kD; e += 128) {
        const int r = e / kD, d = e % kD, i = i0 + r;
        const size_t idx = ((size_t)b * s.Lq + (i < s.Lq ? i : 0)) * qrow + (size_t)h * kD + d;
        qs[r][d] = i < s.Lq ? to_f(q[idx]) : 0.f;
        dos[r][d] = i < s.Lq ? to_f(dout[idx]) : 0.f;
    }
    float L[4], Dv[4], a0[4], a1[4];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int i = i0 + warp * 4 + rr;
        const size_t li = ((size_t)b * s.Hq + h) * s.Lq + (i < s.Lq ? i : 0);
        L[rr] = lse[li];
        Dv[rr] = Drow[li];
        a0[rr] = 0.f;
        a1[rr] = 0.f;
    }
    const int ilast = min(i0 + 15, s.Lq - 1);
    const long pmin = i0 + off, pmax = ilast + off;
    const long lo = s.window > 0 ? max(0L, pmin - s.window + 1) : 0L;
    const long hi = min((long)s.Lk, pmax + 1);
    for (long j0 = (lo / 32) * 32; j0 < hi; j0 += 32) {
        __syncthreads();
        for (int e = tid; e < 32 * kD; e += 128) {
            const int r = e / kD, d = e % kD;
            const long j = j0 + r;
            const bool in = j < s.Lk;
            const size_t idx = ((size_t)b * s.Lk + (in ? j : 0)) * krow + (size_t)g * kD + d;
            ks[r][d] = in ? to_f(k[idx]) : 0.f;
            vs[r][d] = in ? to_f(v[idx]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const int r = warp * 4 + rr, i = i0 + r;
            if (i >= s.Lq || L[rr] == -INFINITY) continue;
            const long p = i + off, j = j0 + lane;
            float sc = 0.f, dp = 0.f;
#pragma unroll 16
            for (int d = 0; d < kD; ++d) {
                sc = fmaf(qs[r][d], ks[lane][d], sc);
                dp = fmaf(dos[r][d], vs[lane][d], dp);
            }
            const bool vis = visible(j, p, s.window, s.Lk);
            const float P = vis ? expf(sc * s.scale - L[rr]) : 0.f;
            const float dS = P * (dp - Dv[rr]);
#pragma unroll 8
            for (int jj = 0; jj < 32; ++jj) {
                const float w = __shfl_sync(0xffffffffu, dS, jj);
                a0[rr] = fmaf(w, ks[jj][lane], a0[rr]);
                a1[rr] = fmaf(w, ks[jj][lane + 32], a1[rr]);
            }
        }
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int i = i0 + warp * 4 + rr;
        if (i >= s.Lq) continue;
        T *row = dq + ((size_t)b * s.Lq + i) * qrow + (size_t)h * kD;
        row[lane] = from_f<T>(a0[rr] * s.scale);
        row[lane + 32] = from_f<T>(a1[rr] * s.scale);
    }
}

// (3) dk, dv: CTA = 32 keys of one KV head (4 warps x 8 keys); loops over the
// group's query heads and the 32-row tiles that can see these keys.
template <typename T>
__global__ void __launch_bounds__(128) bwd_dkdv_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                       const T *__restrict__ v, const T *__restrict__ dout,
                                                       const float *__restrict__ lse,
                                                       const float *__restrict__ Drow, T *__restrict__ dk,
                                                       T *__restrict__ dv, AttnShape s)
{
    __shared__ float Qs[32][kD + 1], dOs[32][kD + 1];
    __shared__ float Ks[32][kD], Vs[32][kD];
    __shared__ float Ls[32], Dsh[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int j0 = blockIdx.x * 32, g = blockIdx.y, b = blockIdx.z;
    const int G = s.Hq / s.Hkv;
    const long off = (long)s.Lk - s.Lq;
    const size_t qrow = (size_t)s.Hq * kD, krow = (size_t)s.Hkv * kD;
    for (int e = tid; e < 32 * kD; e += 128) {
        const int r = e / kD, d = e % kD, j = j0 + r;
        const size_t idx = ((size_t)b * s.Lk + (j < s.Lk ? j : 0)) * krow + (size_t)g * kD + d;
        Ks[r][d] = j < s.Lk ? to_f(k[idx]) : 0.f;
        Vs[r][d] = j < s.Lk ? to_f(v[idx]) : 0.f;
    }
    float dk0[8], dk1[8], dv0[8], dv1[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) dk0[t] = dk1[t] = dv0[t] = dv1[t] = 0.f;
    const int jlast = min(j0 + 31, s.Lk - 1);
    // rows i whose position p = i + off can see some key in [j0, jlast]
    long ilo = (long)j0 - off;
    long ihi = s.window > 0 ? (long)jlast + s.window - 1 - off : (long)s.Lq - 1;
    ilo = max(ilo, 0L);
    ihi = min(ihi, (long)s.Lq - 1);
    for (int h = g * G; h < (g + 1) * G; ++h) {
        for (long i0 = (ilo / 32) * 32; i0 <= ihi; i0 += 32) {
            __syncthreads();
            for (int e = tid; e < 32 * kD; e += 128) {
                const int r = e / kD, d = e % kD;
                const long i = i0 + r;
                const bool in = i < s.Lq;
                const size_t idx = ((size_t)b * s.Lq + (in ? i : 0)) * qrow + (size_t)h * kD + d;
                Qs[r][d] = in ? to_f(q[idx]) : 0.f;
                dOs[r][d] = in ? to_f(dout[idx]) : 0.f;
            }
            if (tid < 32) {
                const long i = i0 + tid;
                const size_t li = ((size_t)b * s.Hq + h) * s.Lq + (i < s.Lq ? i : 0);
                Ls[tid] = i < s.Lq ? lse[li] : -INFINITY;
                Dsh[tid] = i < s.Lq ? Drow[li] : 0.f;
            }
            __syncthreads();
            const long i = i0 + lane, p = i + off;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int kr = warp * 8 + t, j = j0 + kr;
                float sc = 0.f, dp = 0.f;
#pragma unroll 16
                for (int d = 0; d < kD; ++d) {
                    sc = fmaf(Qs[lane][d], Ks[kr][d], sc);
                    dp = fmaf(dOs[lane][d], Vs[kr][d], dp);
                }
                const bool vis = i < s.Lq && Ls[lane] != -INFINITY && visible(j, p, s.window, s.Lk);
                const float P = vis ? expf(sc * s.scale - Ls[lane]) : 0.f;
                const float dS = P * (dp - Dsh[lane]);
#pragma unroll 8
                for (int rr = 0; rr < 32; ++rr) {
                    const float wp = __shfl_sync(0xffffffffu, P, rr);
                    const float ws = __shfl_sync(0xffffffffu, dS, rr);
                    dv0[t] = fmaf(wp, dOs[rr][lane], dv0[t]);
                    dv1[t] = fmaf(wp, dOs[rr][lane + 32], dv1[t]);
                    dk0[t] = fmaf(ws, Qs[rr][lane], dk0[t]);
                    dk1[t] = fmaf(ws, Qs[rr][lane + 32], dk1[t]);
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const int j = j0 + warp * 8 + t;
        if (j >= s.Lk) continue;
        const size_t base = ((size_t)b * s.Lk + j) * krow + (size_t)g * kD;
        dk[base + lane] = from_f<T>(dk0[t] * s.scale);
        dk[base + lane + 32] = from_f<T>(dk1[t] * s.scale);
        dv[base + lane] = from_f<T>(dv0[t]);
        dv[base + lane + 32] = from_f<T>(dv1[t]);
    }
}

// (4) dsinks[h] = sum of its B*Lq terms, fixed order (deterministic).
__global__ void __launch_bounds__(256) dsink_reduce_kernel(const float *__restrict__ terms,
                                                           float *__restrict__ dsinks, long n)
{
    __shared__ float red[256];
    const int h = blockIdx.x, t = threadIdx.x;
    const float *row = terms + (size_t)h * n;
    float acc = 0.f;
    for (long e = t; e < n; e += 256) acc += row[e];
    red[t] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (t < w) red[t] += red[t + w];
        __syncthreads();
    }
    if (t == 0) dsinks[h] = red[0];
}

// ------------------------------------------------------------------ decode
// CTA = (chunk c, query head h, sequence b); 4 warps take 32-key tiles round
// robin; partial state (m, l, o) is kept in the log2 domain.
template <typename T>
__global__ void __launch_bounds__(128) decode_simt_kernel(const T *__restrict__ q, const T *__restrict__ kc,
                                                          const T *__restrict__ vc, const int *__restrict__ seqlens,
                                                          const float *__restrict__ sinks, T *__restrict__ out,
                                                          float *__restrict__ lse, float *__restrict__ ws_o,
                                                          float *__restrict__ ws_ml, DecodeShape s)
{
    __shared__ float qsh[kD];
    __shared__ float ks[4][32][kD + 1];
    __shared__ float red_m[4], red_l[4], red_o[4][kD];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int G = s.Hq / s.Hkv, g = h / G;
    const int len = min(max(seqlens[b], 1), s.Lmax);
    const int lo = s.window > 0 ? max(0, len - s.window) : 0;
    const int nsplit = (len - lo + s.chunk - 1) / s.chunk;
    if (c >= nsplit) return;
    const int kbeg = lo + c * s.chunk, kend = min(len, kbeg + s.chunk);
    const size_t krow = (size_t)s.Hkv * kD;
    const float C = s.scale * kLog2e;
    if (tid < kD) qsh[tid] = to_f(q[((size_t)b * s.Hq + h) * kD + tid]);
    __syncthreads();
    float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
    for (int j0 = kbeg + warp * 32; j0 < kend; j0 += 128) {
        __syncwarp();
        for (int e = lane; e < 32 * kD; e += 32) {
            const int r = e / kD, d = e % kD, j = j0 + r;
            const bool in = j < kend;
            const size_t idx = ((size_t)b * s.Lmax + (in ? j : kbeg)) * krow + (size_t)g * kD + d;
            ks[warp][r][d] = in ? to_f(kc[idx]) : 0.f;
        }
        __syncwarp();
        const int j = j0 + lane;
        float sc = 0.f;
#pragma unroll 16
        for (int d = 0; d < kD; ++d) sc = fmaf(qsh[d], ks[warp][lane][d], sc);
        sc = j < kend ? sc * C : -INFINITY;
        const float mn = fmaxf(m, warp_max(sc));
        const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - mn);
        const float pj = j < kend ? exp2f(sc - mn) : 0.f;
        l = l * alpha + warp_sum(pj);
        o0 *= alpha;
        o1 *= alpha;
        const int nj = min(32, kend - j0);  // V rows past the chunk are never read
        for (int jj = 0; jj < nj; ++jj) {
            const float w = __shfl_sync(0xffffffffu, pj, jj);
            const T *vrow = vc + ((size_t)b * s.Lmax + j0 + jj) * krow + (size_t)g * kD;
            o0 = fmaf(w, to_f(vrow[lane]), o0);
            o1 = fmaf(w, to_f(vrow[lane + 32]), o1);
        }
        m = mn;
    }
    if (lane == 0) {
        red_m[warp] = m;
        red_l[warp] = l;
    }
    red_o[warp][lane] = o0;
    red_o[warp][lane + 32] = o1;
    __syncthreads();
    if (warp != 0) return;
    float M = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
    float Lsum = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const float f = (red_m[w] == -INFINITY) ? 0.f : exp2f(red_m[w] - M);
        Lsum += f * red_l[w];
        a0 += f * red_o[w][lane];
        a1 += f * red_o[w][lane + 32];
    }
    if (nsplit == 1) {
        // the only chunk: fold the sink in here
        const float sk = sinks[h] * kLog2e;
        const float M2 = fmaxf(M, sk);
        const float fo = (M == -INFINITY) ? 0.f : exp2f(M - M2);
        const float fs = (sk == -INFINITY) ? 0.f : exp2f(sk - M2);
        const float Lt = Lsum * fo + fs;
        const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
        T *orow = out + ((size_t)b * s.Hq + h) * kD;
        orow[lane] = from_f<T>(a0 * fo * inv);
        orow[lane + 32] = from_f<T>(a1 * fo * inv);
        if (lane == 0) lse[(size_t)b * s.Hq + h] = Lt > 0.f ? (M2 + log2f(Lt)) * kLn2 : -INFINITY;
    } else {
        const size_t slot = ((size_t)b * s.Hq + h) * s.splits + c;
        ws_o[slot * kD + lane] = a0;
        ws_o[slot * kD + lane + 32] = a1;
        if (lane == 0) {
            ws_ml[slot * 2 + 0] = M;
            ws_ml[slot * 2 + 1] = Lsum;
        }
    }
}

// One warp per (b, h): M = max(sink, max_c m_c), L = 2^(sink-M) + sum_c l_c 2^(m_c-M),
// o = sum_c 2^(m_c-M) o_c / L, lse = (M + log2 L) ln 2.  The sink enters once.
template <typename T>
__global__ void __launch_bounds__(128) decode_combine_kernel(const int *__restrict__ seqlens,
                                                             const float *__restrict__ sinks, T *__restrict__ out,
                                                             float *__restrict__ lse,
                                                             const float *__restrict__ ws_o,
                                                             const float *__restrict__ ws_ml, DecodeShape s)
{
    grid_dep_wait();  // the split partials of the decode grid ahead (programmatic dependent launch)
    const int lane = threadIdx.x & 31;
    const long bh = (long)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (bh >= (long)s.B * s.Hq) return;
    const int b = (int)(bh / s.Hq), h = (int)(bh % s.Hq);
    const int len = min(max(seqlens[b], 1), s.Lmax);
    int lo, lo_al, nsplit;
    decode_range(s, len, lo, lo_al, nsplit);
    if (nsplit <= 1) return;  // written directly by the split kernel
    const size_t slot0 = (size_t)bh * s.splits;
    const float mc = lane < nsplit ? ws_ml[(slot0 + lane) * 2 + 0] : -INFINITY;
    const float lc = lane < nsplit ? ws_ml[(slot0 + lane) * 2 + 1] : 0.f;
    const float sk = sinks[h] * kLog2e;
    const float M = fmaxf(warp_max(mc), sk);
    float Lt = warp_sum((mc == -INFINITY || M == -INFINITY) ? 0.f : lc * exp2f(mc - M));
    Lt += (sk == -INFINITY || M == -INFINITY) ? 0.f : exp2f(sk - M);
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
    float a0 = 0.f, a1 = 0.f;
    for (int c = 0; c < nsplit; ++c) {
        const float m_c = __shfl_sync(0xffffffffu, mc, c);
        const float f = (m_c == -INFINITY) ? 0.f : exp2f(m_c - M);
        a0 = fmaf(f, ws_o[(slot0 + c) * kD + lane], a0);
        a1 = fmaf(f, ws_o[(slot0 + c) * kD + lane + 32], a1);
    }
    T *orow = out + (size_t)bh * kD;
    orow[lane] = from_f<T>(a0 * inv);
    orow[lane + 32] = from_f<T>(a1 * inv);
    if (lane == 0) lse[bh] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
}

}  // namespace

template <typename T>
cudaError_t launch_fwd_simt(const T *q, const T *k, const T *v, const float *sinks, T *out, float *lse,
                            const AttnShape &s, cudaStream_t st)
{
    dim3 grid((s.Lq + 15) / 16, s.Hq, s.B);
    fwd_simt_kernel<T><<<grid, 128, 0, st>>>(q, k, v, sinks, out, lse, s);
    return cudaGetLastError();
}

size_t bwd_simt_workspace_bytes(const AttnShape &s)
{
    const size_t rows = (size_t)s.B * s.Hq * s.Lq;
    return 2 * rows * sizeof(float);
}

template <typename T>
cudaError_t launch_bwd_simt(const T *q, const T *k, const T *v, const float *sinks, const T *out,
                            const T *dout, const float *lse, T *dq, T *dk, T *dv, float *dsinks,
                            const AttnShape &s, void *ws, cudaStream_t st)
{
    const size_t rows = (size_t)s.B * s.Hq * s.Lq;
    float *Drow = static_cast<float *>(ws);
    float *terms = Drow + rows;
    bwd_pre_kernel<T><<<(unsigned)((rows + PreRows<T>::kRowsPerCta - 1) / PreRows<T>::kRowsPerCta), 256, 0, st>>>(
        out, dout, lse, sinks, Drow, terms, nullptr, s);
    bwd_dq_kernel<T><<<dim3((s.Lq + 15) / 16, s.Hq, s.B), 128, 0, st>>>(q, k, v, dout, lse, Drow, dq, s);
    bwd_dkdv_kernel<T><<<dim3((s.Lk + 31) / 32, s.Hkv, s.B), 128, 0, st>>>(q, k, v, dout, lse, Drow, dk, dv, s);
    dsink_reduce_kernel<<<s.Hq, 256, 0, st>>>(terms, dsinks, (long)s.B * s.Lq);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_rows(const T *out, const T *dout, const float *lse, const float *sinks, float *Drow,
                            float *terms, float *zero_rows, const AttnShape &s, cudaStream_t st)
{
    const size_t rows = (size_t)s.B * s.Hq * s.Lq;
    const size_t ctas = (rows + PreRows<T>::kRowsPerCta - 1) / PreRows<T>::kRowsPerCta;
    if (ctas > 0x7fffffffu) return cudaErrorInvalidValue;
    bwd_pre_kernel<T><<<(unsigned)ctas, 256, 0, st>>>(out, dout, lse, sinks, Drow, terms, zero_rows, s);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_decode_simt(const T *q, const T *kc, const T *vc, const int *seqlens, const float *sinks,
                               T *out, float *lse, const DecodeShape &s, float *ws_o, float *ws_ml,
                               cudaStream_t st)
{
    decode_simt_kernel<T><<<dim3(s.splits, s.Hq, s.B), 128, 0, st>>>(q, kc, vc, seqlens, sinks, out, lse, ws_o,
                                                                     ws_ml, s);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_decode_combine(const int *seqlens, const float *sinks, T *out, float *lse,
                                  const DecodeShape &s, const float *ws_o, const float *ws_ml, cudaStream_t st)
{
    const long n = (long)s.B * s.Hq;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine_kernel<T>, seqlens, sinks, out, lse, ws_o, ws_ml, s);
}

#define ATTN_SINK_INSTANTIATE(T)                                                                              \
    template cudaError_t launch_fwd_simt<T>(const T *, const T *, const T *, const float *, T *, float *,     \
                                            const AttnShape &, cudaStream_t);                                 \
    template cudaError_t launch_bwd_simt<T>(const T *, const T *, const T *, const float *, const T *,        \
                                            const T *, const float *, T *, T *, T *, float *,                 \
                                            const AttnShape &, void *, cudaStream_t);                         \
    template cudaError_t launch_bwd_rows<T>(const T *, const T *, const float *, const float *, float *, float *, \
                                            float *, const AttnShape &, cudaStream_t);                                 \
    template cudaError_t launch_decode_simt<T>(const T *, const T *, const T *, const int *, const float *,   \
                                               T *, float *, const DecodeShape &, float *, float *,           \
                                               cudaStream_t);                                                 \
    template cudaError_t launch_decode_combine<T>(const int *, const float *, T *, float *,                   \
                                                  const DecodeShape &, const float *, const float *,          \
                                                  cudaStream_t);
ATTN_SINK_INSTANTIATE(float)
ATTN_SINK_INSTANTIATE(__nv_bfloat16)

}  // namespace attn_sink
