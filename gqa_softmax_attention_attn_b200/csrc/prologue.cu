// prologue.cu -- the step just before attention: the QKV projection's output
// gets its bias, q and k are rotated by YaRN-scaled rotary position embeddings,
// and the three are written in the layouts the attention calls read
// ("GPT-OSS on day 0", section "Attention: GQA with Attention Sinks": the QKV
// projections carry biases and positions use YaRN encoding, as in DeepSeek-V3;
// "GPT-OSS-120B 4-bit ...", section 3: YaRN-type RoPE scaling extends the
// context to 131072 tokens).
//
// Per token t at position p, with frequencies for pair i (D/2 pairs):
//   f_i    = base^(-2i/D)                             (plain rotary frequency)
//   lo, hi = the dimensions where a full wavelength fits beta_fast and
//            beta_slow times into the original context L0:
//            d(n) = D ln(L0 / (2 pi n)) / (2 ln base)
//   e_i    = 1 - clamp((i - lo) / (hi - lo), 0, 1)    (1: keep f_i, 0: interpolate)
//   f'_i   = f_i e_i + (f_i / factor) (1 - e_i)
//   a      = 0.1 ln(factor) + 1 (1 when factor <= 1), multiplying cos and sin
//   rotate-half pairs (i, i + D/2) or interleaved pairs (2i, 2i + 1):
//   x'_lo = a (x_lo cos(p f'_i) - x_hi sin(p f'_i)),  x'_hi = a (x_hi cos + x_lo sin)
// v only gets its bias.  The angles are formed and their sine and cosine taken
// in fp64 (positions up to 131072 times frequencies near 1 leave fp32 with too
// few bits of phase).
//
// Design: HBM-bound (one read and one write of the QKV rows).  The D/2 pair
// frequencies are computed once, on the host, and passed in; a CTA takes
// eight tokens: one fp64 angle per thread into shared memory, then all
// threads move 16-byte chunks of q, k and v (bias as 16-byte vectors too),
// eight pairs (or eight v values) per thread-step.  k and v rows can be written to
// any row of their outputs (kv_rows), which appends them to a decode cache in
// the same pass.
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

constexpr int kD = 64;
constexpr int kPairs = kD / 2;
constexpr int kThreads = 256;

struct ProParams {
    const __nv_bfloat16 *__restrict__ qkv;  // [T, (Hq + 2 Hkv) * D]
    const float *bias;         // [(Hq + 2 Hkv) * D] or nullptr
    const int *pos;            // [T]
    const int *kv_rows;        // [T] or nullptr (row t)
    __nv_bfloat16 *__restrict__ q, *__restrict__ k, *__restrict__ v;
    int T, Hq, Hkv, interleaved;
    int kv_rows_total;         // rows of k / v (a kv_rows entry outside [0, rows) writes nothing)
    double attn_factor;
    double freq[kPairs];       // rotary frequency of each pair after the YaRN correction
};

// rotary frequency of pair i after the YaRN correction (host, once per call)
double yarn_freq(const RopeParams &r, int i)
{
    const double f = pow(r.base, -2.0 * i / kD);
    if (!(r.factor > 1.0)) return f;
    const double lo = kD * log(r.original_max_pos / (2.0 * M_PI * r.beta_fast)) / (2.0 * log(r.base));
    const double hi = kD * log(r.original_max_pos / (2.0 * M_PI * r.beta_slow)) / (2.0 * log(r.base));
    double ramp = hi > lo ? (i - lo) / (hi - lo) : (i >= lo ? 1.0 : 0.0);
    ramp = ramp < 0.0 ? 0.0 : (ramp > 1.0 ? 1.0 : ramp);
    const double keep = 1.0 - ramp;
    return f * keep + (f / r.factor) * (1.0 - keep);
}

// 8 consecutive fp32 bias values (16-byte aligned)
__device__ __forceinline__ void bias8(const float *b, float (&x)[8])
{
    const float4 u = *reinterpret_cast<const float4 *>(b), w = *reinterpret_cast<const float4 *>(b + 4);
    x[0] += u.x; x[1] += u.y; x[2] += u.z; x[3] += u.w;
    x[4] += w.x; x[5] += w.y; x[6] += w.z; x[7] += w.w;
}

__device__ __forceinline__ float2 bf2(uint32_t w)
{
    const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w);
    return __bfloat1622float2(h);
}

// One 8-pair (or, for v, 8-value) step of token tt's row.
__device__ __forceinline__ void prologue_step(const ProParams &p, int t, int u, const float *cs, const float *sn)
{
    const int width = (p.Hq + 2 * p.Hkv) * kD;
    const int rot_units = (p.Hq + p.Hkv) * (kPairs / 8);
    const __nv_bfloat16 *__restrict__ row = p.qkv + (size_t)t * width;
    const int kr = p.kv_rows ? p.kv_rows[t] : t;
    const bool kv_ok = kr >= 0 && kr < p.kv_rows_total;
    if (u < rot_units) {
        // rotated heads (q then k): pairs i0 .. i0 + 7 of head h
        const int h = u / (kPairs / 8), i0 = (u % (kPairs / 8)) * 8;
        if (h >= p.Hq && !kv_ok) return;
        const int col = h * kD;
        float xa[8], xb[8];
        if (!p.interleaved) {
            const uint4 a = *reinterpret_cast<const uint4 *>(row + col + i0);
            const uint4 b = *reinterpret_cast<const uint4 *>(row + col + kPairs + i0);
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 fa = bf2(aw[j]), fb = bf2(bw[j]);
                xa[2 * j] = fa.x;
                xa[2 * j + 1] = fa.y;
                xb[2 * j] = fb.x;
                xb[2 * j + 1] = fb.y;
            }
        } else {
            const uint4 a = *reinterpret_cast<const uint4 *>(row + col + 2 * i0);
            const uint4 b = *reinterpret_cast<const uint4 *>(row + col + 2 * i0 + 8);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 f = bf2(w[j]);
                xa[j] = f.x;
                xb[j] = f.y;
            }
        }
        if (p.bias) {
            if (!p.interleaved) {
                bias8(p.bias + col + i0, xa);
                bias8(p.bias + col + kPairs + i0, xb);
            } else {
                float bb[2][8] = {};
                bias8(p.bias + col + 2 * i0, bb[0]);
                bias8(p.bias + col + 2 * i0 + 8, bb[1]);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    xa[j] += bb[j >> 2][2 * (j & 3)];
                    xb[j] += bb[j >> 2][2 * (j & 3) + 1];
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float c = cs[i0 + j], sv = sn[i0 + j];
            const float ra = xa[j] * c - xb[j] * sv;
            const float rb = xb[j] * c + xa[j] * sv;
            xa[j] = ra;
            xb[j] = rb;
        }
        __nv_bfloat16 *__restrict__ dst =
            h < p.Hq ? p.q + ((size_t)t * p.Hq + h) * kD : p.k + ((size_t)kr * p.Hkv + (h - p.Hq)) * kD;
        if (!p.interleaved) {
            uint32_t oa[4], ob[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                oa[j] = pack_bf16x2(xa[2 * j], xa[2 * j + 1]);
                ob[j] = pack_bf16x2(xb[2 * j], xb[2 * j + 1]);
            }
            *reinterpret_cast<uint4 *>(dst + i0) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
            *reinterpret_cast<uint4 *>(dst + kPairs + i0) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
        } else {
            uint32_t oi[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) oi[j] = pack_bf16x2(xa[j], xb[j]);
            *reinterpret_cast<uint4 *>(dst + 2 * i0) = make_uint4(oi[0], oi[1], oi[2], oi[3]);
            *reinterpret_cast<uint4 *>(dst + 2 * i0 + 8) = make_uint4(oi[4], oi[5], oi[6], oi[7]);
        }
    } else {
        // v: bias only, values d0 .. d0 + 7 of head h
        if (!kv_ok) return;
        const int vu = u - rot_units;
        const int h = vu / (kD / 8), d0 = (vu % (kD / 8)) * 8;
        const int col = (p.Hq + p.Hkv + h) * kD + d0;
        const uint4 a = *reinterpret_cast<const uint4 *>(row + col);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
        float x[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = bf2(w[j]);
            x[2 * j] = f.x;
            x[2 * j + 1] = f.y;
        }
        if (p.bias) bias8(p.bias + col, x);
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = pack_bf16x2(x[2 * j], x[2 * j + 1]);
        *reinterpret_cast<uint4 *>(p.v + ((size_t)kr * p.Hkv + h) * kD + d0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// kTok tokens per CTA: the (token, pair) angles' sines and cosines into shared
// memory, then every thread moves 16-byte chunks of the tokens' rows
// (measured on 4096 tokens of gpt-oss-20b: 4, 8, 16 tokens per CTA 27, 26, 33 us;
// unrolling the copy loop by 4 instead of 2 changed nothing)
constexpr int kTok = 8;

__global__ void __launch_bounds__(kThreads) prologue_kernel(const ProParams p)
{
    __shared__ float cs[kTok][kPairs], sn[kTok][kPairs];
    const int t0 = blockIdx.x * kTok;
    for (int a = threadIdx.x; a < kTok * kPairs; a += kThreads) {
        const int tt = a / kPairs, i = a % kPairs;
        if (t0 + tt < p.T) {
            double sv, cv;
            sincos((double)p.pos[t0 + tt] * p.freq[i], &sv, &cv);
            cs[tt][i] = (float)(cv * p.attn_factor);
            sn[tt][i] = (float)(sv * p.attn_factor);
        }
    }
    __syncthreads();
    const int units = (p.Hq + p.Hkv) * (kPairs / 8) + p.Hkv * (kD / 8);
    const int ntok = min(kTok, p.T - t0);
#pragma unroll 2
    for (int x = threadIdx.x; x < ntok * units; x += kThreads) {
        const int tt = x / units;
        prologue_step(p, t0 + tt, x - tt * units, cs[tt], sn[tt]);
    }
}

}  // namespace

cudaError_t launch_qkv_prologue(const void *qkv, const float *bias, const int *positions, const int *kv_rows,
                                void *q, void *k, void *v, int T, int Hq, int Hkv, int kv_rows_total,
                                const RopeParams &r, cudaStream_t st)
{
    ProParams p;
    p.qkv = static_cast<const __nv_bfloat16 *>(qkv);
    p.bias = bias;
    p.pos = positions;
    p.kv_rows = kv_rows;
    p.q = static_cast<__nv_bfloat16 *>(q);
    p.k = static_cast<__nv_bfloat16 *>(k);
    p.v = static_cast<__nv_bfloat16 *>(v);
    p.T = T;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.interleaved = r.interleaved;
    p.kv_rows_total = kv_rows_total;
    p.attn_factor = r.factor > 1.0 ? 0.1 * log(r.factor) + 1.0 : 1.0;
    for (int i = 0; i < kPairs; ++i) p.freq[i] = yarn_freq(r, i);
    prologue_kernel<<<(T + kTok - 1) / kTok, kThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace attn_sink
