// fwd_tc.cu -- bf16 prefill forward of sink-softmax GQA attention on the
// sm_100a tensor cores (tcgen05, accumulators in tensor memory, TMA-staged
// operands).
//
// What it computes ("GPT-OSS on day 0", sections "Attention: GQA with
// Attention Sinks" and "Sink Attention"): per query row, the online softmax
// whose running maximum is seeded with the head's sink logit (and whose
// running sum is seeded with the sink's own mass, 1), over the visible keys of
// a dense causal or window-banded causal layer; O = sum_j p_j v_j / l and the
// log-sum-exp including the sink.
//
// Design (B200):
//  * CTA tile = 128 query rows = (128 / Gp) positions x Gp query heads of one
//    KV group, so every K/V tile fetched is shared by Gp heads (GQA packing;
//    no cluster multicast).  Q is loaded once by a 4-D TMA box.
//  * Warp 0: TMA producer (K and V tiles of BN keys into an NS-stage ring).
//    Warp 1: allocates tensor memory and issues tcgen05.mma from one thread:
//    S = Q K^T into a double-buffered TMEM tile, O += P V with P read from
//    TMEM.  Warps 2-5: one thread per row -- tcgen05.ld of S, masking, the
//    exp2 softmax, P written back over S as bf16, conditional rescale of O.
//  * The running maximum used for the exponentials is only moved when the
//    true maximum exceeds it by more than 2^8, so the O rescale (which must
//    wait for the previous PV product) is rare; the result is exact either
//    way because numerator and denominator share the same reference.
//  * Causal / band tile skipping: only KV tiles that intersect the rows'
//    visible ranges are visited; element masks are applied only on tiles a
//    row does not see entirely.
//  * Every wait is bounded (globaltimer); on expiry the CTA raises a status
//    bit, waits (bounded) for its own TMA loads and MMAs, frees tensor memory
//    and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

constexpr int kM = 128;
constexpr int kD = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int BN, int NS>
struct FwdCfg {
    static constexpr int kQBytes = kM * kD * 2;
    static constexpr int kKVBytes = BN * kD * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffV = kOffK + NS * kKVBytes;
    static constexpr int kOffBar = kOffV + NS * kKVBytes;
    // q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2], p_full[2], o_done, drain
    static constexpr int kNumBar = 1 + 4 * NS + 2 + 2 + 1 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBar * 8;
    static constexpr int kTmemCols = (2 * BN + kD <= 256) ? 256 : 512;
    // + slack for 1024-byte alignment; a CTA that takes all 512 TMEM columns
    // also takes enough shared memory that no second CTA lands on its SM
    static constexpr int kSmemUsed = kOffMisc + 16 + 1024;
    static constexpr int kSmemBytes = (kTmemCols == 512 && kSmemUsed < 116 * 1024) ? 116 * 1024 : kSmemUsed;
    static constexpr int kTmS0 = 0;
    static constexpr int kTmO = 2 * BN;
};

struct FwdTcParams {
    int B, Lq, Lk, Hq, Hkv, window;
    int G, Gp, P;  // group size, query heads packed per tile, positions per tile
    int n_ptiles;
    float c_log2;  // scale * log2(e)
    const float *sinks;
    __nv_bfloat16 *out;
    float *lse;
    unsigned *status;
    long long timeout_ns;
};

__device__ __forceinline__ bool wait_noabort(uint64_t *bar, uint32_t parity, unsigned *status, long long tmo)
{
    int never = 0;
    return mbar_wait(bar, parity, &never, status, tmo);
}

template <int BN, int NS>
__global__ void __launch_bounds__(192, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdTcParams p)
{
    using Cfg = FwdCfg<BN, NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;
    uint64_t *k_empty = k_full + NS;
    uint64_t *v_full = k_empty + NS;
    uint64_t *v_empty = v_full + NS;
    uint64_t *s_full = v_empty + NS;
    uint64_t *p_full = s_full + 2;
    uint64_t *o_done = p_full + 2;
    uint64_t *drain = o_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Cfg::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = p.n_ptiles - 1 - (int)blockIdx.x;  // longest causal tiles first
    const int h0 = (int)blockIdx.y * p.Gp;
    const int b = (int)blockIdx.z;
    const int g = h0 / p.G;
    const int pos0 = qt * p.P;
    const long off = (long)p.Lk - p.Lq;
    const int pos_last = min(pos0 + p.P - 1, p.Lq - 1);
    const long lo = p.window > 0 ? max(0L, pos0 + off - p.window + 1) : 0L;
    const long hi = min((long)p.Lk, pos_last + off + 1);  // exclusive
    const int t_lo = (int)(lo / BN);
    const int n_tiles = hi > lo ? (int)((hi - 1) / BN) - t_lo + 1 : 0;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 128);
        }
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n_tiles > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            uint32_t k_issued[NS], v_issued[NS];
            for (int s = 0; s < NS; ++s) k_issued[s] = v_issued[s] = 0;
            mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
            tma_load_4d(smem + Cfg::kOffQ, &tmQ, 0, h0, pos0, b, q_full);
            for (int jt = 0; jt < n_tiles; ++jt) {
                const int st = jt % NS;
                const uint32_t ph = (uint32_t)(jt / NS) & 1u;
                const int j0 = (t_lo + jt) * BN;
                if (!mbar_wait(&k_empty[st], ph ^ 1u, abort_flag, p.status, p.timeout_ns)) break;
                mbar_arrive_expect_tx(&k_full[st], Cfg::kKVBytes);
                tma_load_4d(smem + Cfg::kOffK + st * Cfg::kKVBytes, &tmK, 0, g, j0, b, &k_full[st]);
                ++k_issued[st];
                if (!mbar_wait(&v_empty[st], ph ^ 1u, abort_flag, p.status, p.timeout_ns)) break;
                mbar_arrive_expect_tx(&v_full[st], Cfg::kKVBytes);
                tma_load_4d(smem + Cfg::kOffV + st * Cfg::kKVBytes, &tmV, 0, g, j0, b, &v_full[st]);
                ++v_issued[st];
            }
            // every load issued must land before the CTA may exit
            wait_noabort(q_full, 0, p.status, p.timeout_ns);
            for (int s = 0; s < NS; ++s) {
                if (k_issued[s]) wait_noabort(&k_full[s], (k_issued[s] - 1) & 1u, p.status, p.timeout_ns);
                if (v_issued[s]) wait_noabort(&v_full[s], (v_issued[s] - 1) & 1u, p.status, p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            const uint32_t id_s = idesc_bf16_f32(kM, BN, 0);
            const uint32_t id_pv = idesc_bf16_f32(kM, kD, 1);
            const uint32_t q_addr = smem_u32(smem + Cfg::kOffQ);
            const uint32_t k_addr = smem_u32(smem + Cfg::kOffK);
            const uint32_t v_addr = smem_u32(smem + Cfg::kOffV);
            bool ok = mbar_wait(q_full, 0, abort_flag, p.status, p.timeout_ns);
            auto issue_pv = [&](int t) -> bool {
                const int sb = t & 1, st = t % NS;
                const uint32_t ph = (uint32_t)(t / NS) & 1u;
                if (!mbar_wait(&p_full[sb], (uint32_t)(t >> 1) & 1u, abort_flag, p.status, p.timeout_ns))
                    return false;
                if (!mbar_wait(&v_full[st], ph, abort_flag, p.status, p.timeout_ns)) return false;
                tc_fence_after();
                const uint32_t vb = v_addr + st * Cfg::kKVBytes;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // V tile [BN keys][64 d] is the MN-major B operand: 16 keys = 2048 bytes per step
                    const uint64_t bdesc = smem_desc_sw128(vb + kk * 2048, BN * 128, 1024);
                    mma_ts(tmem + Cfg::kTmO, tmem + Cfg::kTmS0 + sb * BN + kk * 8, bdesc, id_pv,
                           (t > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(o_done);
                mma_commit(&v_empty[st]);
                return true;
            };
            if (ok) {
                tc_fence_after();
                for (int jt = 0; jt < n_tiles && ok; ++jt) {
                    const int st = jt % NS, sb = jt & 1;
                    const uint32_t ph = (uint32_t)(jt / NS) & 1u;
                    if (!mbar_wait(&k_full[st], ph, abort_flag, p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t kb = k_addr + st * Cfg::kKVBytes;
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(q_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(kb + kk * 32, 16, 1024);
                        mma_ss(tmem + Cfg::kTmS0 + sb * BN, adesc, bdesc, id_s, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&s_full[sb]);
                    mma_commit(&k_empty[st]);
                    if (jt >= 1) ok = issue_pv(jt - 1);
                }
                if (ok) issue_pv(n_tiles - 1);
            }
            mma_commit(drain);
            wait_noabort(drain, 0, p.status, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int pos = pos0 + r / p.Gp;
        const int h = h0 + r % p.Gp;
        const bool row_valid = pos < p.Lq;
        const long pabs = pos + off;
        const float sink = p.sinks[h];
        const float C = p.c_log2;
        float m = sink * kLog2e;  // reference maximum, log2 units
        float l = (sink == -INFINITY) ? 0.f : 1.f;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        bool ok = true;

        for (int jt = 0; jt < n_tiles; ++jt) {
            const int sb = jt & 1;
            const long j0 = (long)(t_lo + jt) * BN;
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&s_full[sb], (uint32_t)(jt >> 1) & 1u, abort_flag, p.status, p.timeout_ns))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[BN / 32][32];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) tmem_ld32(trow + Cfg::kTmS0 + sb * BN + c * 32, sr[c]);
            tmem_wait_ld();
            float sv[BN];
#pragma unroll
            for (int c = 0; c < BN; ++c) sv[c] = __uint_as_float(sr[c / 32][c % 32]);
            const bool full_vis = (j0 + BN - 1 <= pabs) && (j0 + BN <= p.Lk) &&
                                  (p.window <= 0 || j0 > pabs - p.window);
            if (__any_sync(0xffffffffu, !full_vis)) {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const long j = j0 + c;
                    const bool vis = j <= pabs && j < p.Lk && (p.window <= 0 || j > pabs - p.window);
                    sv[c] = vis ? sv[c] : -INFINITY;
                }
            }
            float tmax = sv[0];
#pragma unroll
            for (int c = 1; c < BN; ++c) tmax = fmaxf(tmax, sv[c]);
            const float m_new = fmaxf(m, tmax * C);
            const bool rescale = m_new > m + kRescaleThreshold;
            const float alpha = rescale ? ((m == -INFINITY) ? 0.f : ex2(m - m_new)) : 1.f;
            if (rescale) m = m_new;
            const float neg_m = (m == -INFINITY) ? 0.f : -m;
            // P (bf16 pairs) overwrites the first BN/2 columns of this S buffer,
            // which has been read in full already; 32 scores per store.
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = ex2(fmaf(sv[32 * c + 2 * e], C, neg_m));
                    const float p1 = ex2(fmaf(sv[32 * c + 2 * e + 1], C, neg_m));
                    sum += p0 + p1;
                    pk[e] = pack_bf16x2(p0, p1);
                }
                tmem_st16(trow + Cfg::kTmS0 + sb * BN + c * 16, pk);
            }
            l = l * alpha + sum;
            if (jt > 0) {
                // O holds sum_{t<jt} P_t V_t once PV(jt-1) completes
                if (!__all_sync(0xffffffffu,
                                mbar_wait(o_done, (uint32_t)(jt - 1) & 1u, abort_flag, p.status, p.timeout_ns))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
                    uint32_t o[2][32];
                    tmem_ld32(trow + Cfg::kTmO, o[0]);
                    tmem_ld32(trow + Cfg::kTmO + 32, o[1]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        o[c / 32][c % 32] = __float_as_uint(__uint_as_float(o[c / 32][c % 32]) * alpha);
                    tmem_st32(trow + Cfg::kTmO, o[0]);
                    tmem_st32(trow + Cfg::kTmO + 32, o[1]);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[sb]);
        }

        // ------------------------------------------------------------ epilogue
        float ov[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) ov[c] = 0.f;
        if (ok && n_tiles > 0) {
            if (__all_sync(0xffffffffu,
                           mbar_wait(o_done, (uint32_t)(n_tiles - 1) & 1u, abort_flag, p.status, p.timeout_ns))) {
                tc_fence_after();
                uint32_t o[2][32];
                tmem_ld32(trow + Cfg::kTmO, o[0]);
                tmem_ld32(trow + Cfg::kTmO + 32, o[1]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 64; ++c) ov[c] = __uint_as_float(o[c / 32][c % 32]);
            } else {
                ok = false;
            }
        }
        if (row_valid && ok) {
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + (((size_t)b * p.Lq + pos) * p.Hq + h) * kD);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 w;
                w.x = pack_bf16x2(ov[8 * c + 0] * inv, ov[8 * c + 1] * inv);
                w.y = pack_bf16x2(ov[8 * c + 2] * inv, ov[8 * c + 3] * inv);
                w.z = pack_bf16x2(ov[8 * c + 4] * inv, ov[8 * c + 5] * inv);
                w.w = pack_bf16x2(ov[8 * c + 6] * inv, ov[8 * c + 7] * inv);
                dst[c] = w;
            }
            p.lse[((size_t)b * p.Hq + h) * p.Lq + pos] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

template <int BN, int NS>
cudaError_t launch_cfg(const void *q, const void *k, const void *v, const float *sinks, void *out, float *lse,
                       const AttnShape &s, cudaStream_t st)
{
    using Cfg = FwdCfg<BN, NS>;
    FwdTcParams p;
    p.B = s.B;
    p.Lq = s.Lq;
    p.Lk = s.Lk;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.window = s.window;
    p.G = s.Hq / s.Hkv;
    int gp = 1;
    while (gp * 2 <= 16 && p.G % (gp * 2) == 0) gp *= 2;
    p.Gp = gp;
    p.P = kM / gp;
    p.n_ptiles = (s.Lq + p.P - 1) / p.P;
    p.c_log2 = s.scale * kLog2e;
    p.sinks = sinks;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = device_status_ptr();
    p.timeout_ns = wait_timeout_ns();

    alignas(64) CUtensorMap mq, mk, mv;
    {
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.Hq, (uint64_t)s.Lq, (uint64_t)s.B};
        const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)s.Hq * kD * 2, (uint64_t)s.Lq * s.Hq * kD * 2};
        const uint32_t box[4] = {(uint32_t)kD, (uint32_t)p.Gp, (uint32_t)p.P, 1u};
        if (!encode_tensor_map_4d(&mq, const_cast<void *>(q), 2, dims, strides, box, true))
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.Hkv, (uint64_t)s.Lk, (uint64_t)s.B};
        const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)s.Hkv * kD * 2, (uint64_t)s.Lk * s.Hkv * kD * 2};
        const uint32_t box[4] = {(uint32_t)kD, 1u, (uint32_t)BN, 1u};
        if (!encode_tensor_map_4d(&mk, const_cast<void *>(k), 2, dims, strides, box, true))
            return cudaErrorInvalidValue;
        if (!encode_tensor_map_4d(&mv, const_cast<void *>(v), 2, dims, strides, box, true))
            return cudaErrorInvalidValue;
    }
    auto kern = fwd_tc_kernel<BN, NS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_ptiles, s.Hq / p.Gp, s.B);
    kern<<<grid, 192, Cfg::kSmemBytes, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace

bool fwd_tc_supported(const AttnShape &s)
{
    if (s.D != kD || s.Hq % s.Hkv != 0) return false;
    if (s.B > 65535 || s.Hq > 65535) return false;
    return true;
}

cudaError_t launch_fwd_tc(const void *q, const void *k, const void *v, const float *sinks, void *out,
                          float *lse, const AttnShape &s, cudaStream_t st)
{
    return launch_cfg<128, 2>(q, k, v, sinks, out, lse, s, st);
}

}  // namespace attn_sink
