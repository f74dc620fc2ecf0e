// bwd_tc.cu -- bf16 backward of sink-softmax GQA attention on the sm_100a
// tensor cores (tcgen05 / TMEM / TMA).
//
// What it computes (derived from the forward's definition -- "GPT-OSS on
// day 0", section "Sink Attention": the sink is one more logit with no value
// row, so it adds nothing to dK, dV or dQ beyond its share of the softmax
// denominator, which the saved log-sum-exp already carries):
//   P_ij  = exp(s_ij - lse_i)            (lse includes the sink)
//   dS_ij = P_ij (<dO_i, v_j> - D_i),    D_i = <dO_i, O_i>
//   dV_j += P_ij dO_i,  dK_j += scale dS_ij q_i,  dQ_i += scale dS_ij k_j
// D_i and dsink are produced by the row kernel in simt_kernels.cu.
//
// Design (B200), one CTA per (128-key tile, KV head g, batch b):
//  * K and V of the tile stay in shared memory; the CTA walks every q tile
//    (128 rows = positions x query heads of the group, as in the forward)
//    that can see a key of the tile.  Q and dO tiles stream in by TMA (two
//    stages); lse and D for the tile's 128 rows go to shared memory.
//  * Warp 1 runs the MMA issue loop as a whole warp (warp-uniform operands),
//    one elected lane issuing: S^T = K Q^T and dP^T = V dO^T (keys as
//    the M dimension, so a thread of the softmax-gradient warps owns a key
//    row); then dV += P^T dO and dK += dS^T Q with P^T and dS^T read back
//    from tensor memory; then dQ = dS K with dS from shared memory (written
//    there in the MN-major layout by the same threads).  S^T of the next q
//    tile is issued as soon as the current S^T has been read, so it overlaps
//    the rest of the gradient pass and the dV / dK / dQ products.
//  * Warps 2-5 and 10-13: two warps per key row (one per 64-column half of
//    the q tile, so each SM sub-partition runs two of them), in two phases:
//    P from S^T (bf16 pairs into their own TMEM columns, releasing S^T), then
//    dS = P (dP - D) from dP^T; dS^T goes back over the half's read columns
//    of dP^T as bf16, dS to shared memory.
//  * With at most 16 positions per q tile the causal / window mask is one
//    more K = 16 step of S^T: a per-key-row table of 0 / -2^100 over the q
//    tile's positions times the one-hot of each column's position.  The load
//    warp writes the table with the tile's lse and D (one per stage), only
//    for q tiles that hide some key, and the MMA warp adds the step only
//    there, so the P pass never tests visibility.
//  * Warps 6-9 move each dQ tile from TMEM to shared memory (two 128-byte-
//    swizzled fp32 halves) and add it into an fp32 dQ accumulator in global
//    memory with TMA reduce-adds (L2 atomics, evict_last so the accumulator
//    stays in L2; the summation order over key tiles is not fixed).  dK and
//    dV of the tile are written once, at the end (deterministic).  A finish
//    kernel turns the accumulator into bf16 dQ and sums dsink in a fixed
//    order; the main and finish kernels are chained to the row pre-pass by
//    programmatic dependent launch.
//  * One CTA per SM (512 TMEM columns); the 14 warps cap registers at 128 per
//    thread.  The grid is 1-D with the key tile slowest, so the causally
//    longest CTAs of every head and batch start first.
//  * Every wait is bounded; on expiry the CTA raises the device status bit,
//    drains its own TMA and MMA work, frees tensor memory and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include <type_traits>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

constexpr int kM = 128;  // keys per tile (rows of the transposed score tile)
constexpr int kD = 64;
constexpr int kThreads = 448;  // 14 warps: loads, MMA, 4 dQ, 8 gradient
constexpr float kLog2e = 1.4426950408889634f;

constexpr int kTile = kM * kD * 2;  // 16 KB bf16 tile
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kTile;
constexpr int kOffQ = kOffV + kTile;       // 2 stages
constexpr int kOffDO = kOffQ + 2 * kTile;  // 2 stages
constexpr int kOffDS = kOffDO + 2 * kTile;  // dS, MN-major: two 64-row atoms of 16 KB
constexpr int kOffStg = kOffDS + 2 * kTile;  // fp32 dQ staging: two [128][32] halves, 128-byte swizzle
constexpr int kOffLD = kOffStg + 128 * 64 * 4;  // [2 stages][lse2 | D][128] fp32
// mask operands of the extra K = 16 step of S^T (no swizzle, K-major; element
// (row, k) at (row / 8) * 256 + (k / 8) * 128 + (row % 8) * 16 + (k % 8) * 2):
// [2 stages] per key row, 0 where the q tile's position k sees the key, else
// -2^100; per q column c, the one-hot of its position c / GP
constexpr int kEBytes = kM * 32;
constexpr int kOffEK = kOffLD + 2 * 2 * 128 * 4;
constexpr int kOffEQ = kOffEK + 2 * kEBytes;
constexpr int kOffBar = kOffEQ + kEBytes;
// kv_full, qdo_full[2], qdo_empty[2], s_full, s_consumed, dp_full, p_ready,
// pt_free, ds_free, dq_full, dq_free, stg_full, stg_free, dkv_done, drain
constexpr int kNumBar = 17;
constexpr int kOffMisc = kOffBar + kNumBar * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
// TMEM columns: S^T | P^T (bf16 pairs) | dP^T | dV | dK | dQ.  dS^T (bf16
// pairs) goes over dP^T: q rows 0-63 at its columns 0-31, rows 64-127 at
// 64-95, each inside the range its own warp has already read.
constexpr int kTmST = 0, kTmPT = 128, kTmDPT = 192, kTmDV = 320, kTmDK = 384, kTmDQ = 448;

struct BwdParams {
    int B, Lq, Lk, Hq, Hkv, window, G;
    int P, n_htiles;  // positions per q tile, head tiles per group
    float c_log2, scale;
    const float *lse, *Drow;
    __nv_bfloat16 *dk, *dv;
    unsigned *status;
    long long timeout_ns;
};

// Drain wait used on the way out (after an abort too): ignores the abort flag
// and allows at least 1 s whatever the caller's wait limit, so a CTA never
// exits with its own TMA loads or MMAs still in flight.
__device__ __forceinline__ bool wait_noabort(uint64_t *bar, uint32_t parity, unsigned *status, long long tmo)
{
    int never = 0;
    return mbar_wait(bar, parity, &never, status, tmo > 1000000000LL ? tmo : 1000000000LL);
}

template <int GP>  // query heads packed per q tile
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmDQ, const BwdParams p)
{
    constexpr int P = kM / GP;  // positions per q tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *kv_full = bars + 0;
    uint64_t *qdo_full = bars + 1;   // [2]
    uint64_t *qdo_empty = bars + 3;  // [2]
    uint64_t *s_full = bars + 5;
    uint64_t *s_consumed = bars + 6;
    uint64_t *dp_full = bars + 7;
    uint64_t *p_ready = bars + 8;
    uint64_t *pt_free = bars + 9;
    uint64_t *ds_free = bars + 10;
    uint64_t *dq_full = bars + 11;
    uint64_t *dq_free = bars + 12;
    uint64_t *stg_full = bars + 13;
    uint64_t *stg_free = bars + 14;
    uint64_t *dkv_done = bars + 15;
    uint64_t *drain = bars + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    float *ld = reinterpret_cast<float *>(smem + kOffLD);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // The launch overlaps the row pre-pass (programmatic dependent launch):
    // the set-up, K, V, Q and dO loads and the first scores need nothing from
    // it; the load warp waits for it before reading D, the dQ warps before
    // their first add into the accumulator it clears.  The finish kernel may
    // start once every CTA of this grid is running.
    grid_dep_launch();
    // 1-D grid, key tile slowest: under a causal mask the first key tiles see
    // the most q tiles, so every head's and batch's longest CTAs start first
    const int per_kt = p.Hkv * p.B;
    const int kt = (int)blockIdx.x / per_kt;
    const int g = ((int)blockIdx.x % per_kt) % p.Hkv, b = ((int)blockIdx.x % per_kt) / p.Hkv;
    const int k0 = kt * kM;
    const long off = (long)p.Lk - p.Lq;
    // query positions whose rows can see a key of [k0, k0 + 128)
    const long pos_lo = max(0L, (long)k0 - off);
    long pos_hi = (long)p.Lq - 1;
    if (p.window > 0) pos_hi = min(pos_hi, (long)k0 + kM - 1 + p.window - 1 - off);
    const int n_q = pos_hi >= pos_lo ? (int)(pos_hi / P - pos_lo / P + 1) : 0;
    const int qt_lo = (int)(pos_lo / P);
    const int n_iter = n_q * p.n_htiles;
    // at most 16 positions per q tile: the mask comes from an extra MMA step
    constexpr bool mask_mma = GP >= 8;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&qdo_full[s], 2);
            mbar_init(&qdo_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_consumed, 256);
        mbar_init(dp_full, 1);
        mbar_init(p_ready, 256);
        mbar_init(pt_free, 1);
        mbar_init(ds_free, 1);
        mbar_init(dq_full, 1);
        mbar_init(dq_free, 128);
        mbar_init(stg_full, 128);
        mbar_init(stg_free, 1);
        mbar_init(dkv_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto iter_head = [&](int i, int &h0, int &pos0) {
        const int ht = i / n_q, qt = qt_lo + i % n_q;
        h0 = g * p.G + ht * GP;
        pos0 = qt * P;
    };
    // does q tile i hide some key of this tile from some of its positions?
    // key j sees positions [max(jrel, 0), jrel + window - 1] of the tile,
    // jrel = j - first position - (Lk - Lq); keys past Lk see none
    auto tile_masked = [&](int i) {
        int h0, pos0;
        iter_head(i, h0, pos0);
        const long jr0 = (long)k0 - pos0 - off;
        return jr0 + kM - 1 > 0 || k0 + kM > p.Lk || (p.window > 0 && jr0 + p.window - 1 < P - 1);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ loads
        uint32_t issued_qdo0 = 0, issued_qdo1 = 0;
        bool ok = true;
        if (lane == 0 && n_iter > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmDO);
            mbar_arrive_expect_tx(kv_full, 2 * kTile);
            tma_load_4d(smem + kOffK, &tmK, 0, g, k0, b, kv_full);
            tma_load_4d(smem + kOffV, &tmV, 0, g, k0, b, kv_full);
        }
        if (mask_mma) {
            // the one-hot of each column's position (covered by the first
            // stage's proxy fence below)
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int c = lane + 32 * (t >> 1), k = 8 * (t & 1);
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    w[u] = (k + 2 * u == c / GP ? 0x3F80u : 0u) | ((k + 2 * u + 1 == c / GP ? 0x3F80u : 0u) << 16);
                *reinterpret_cast<uint4 *>(smem + kOffEQ + (c >> 3) * 256 + (t & 1) * 128 + (c & 7) * 16) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        static_assert(kM == 32 * 4, "one group of 4 lse / D values per lane");
        grid_dep_wait();  // D comes from the pre-pass
        for (int i = 0; i < n_iter && ok; ++i) {
            const int st = i & 1;
            int h0, pos0;
            iter_head(i, h0, pos0);
            // lse and D of the tile, read before the stage is free so that the
            // loads overlap the wait: lane l reads 4 consecutive positions of
            // one head (16-byte loads when aligned)
            const int hl = lane * 4 / P, pl0 = lane * 4 % P;  // head within the tile, first position
            const size_t li0 = ((size_t)b * p.Hq + h0 + hl) * p.Lq + pos0 + pl0;
            float L4[4], D4[4];
            if (pos0 + pl0 + 3 < p.Lq && (li0 & 3) == 0) {
                const float4 a = *reinterpret_cast<const float4 *>(p.lse + li0);
                const float4 d = *reinterpret_cast<const float4 *>(p.Drow + li0);
                L4[0] = a.x; L4[1] = a.y; L4[2] = a.z; L4[3] = a.w;
                D4[0] = d.x; D4[1] = d.y; D4[2] = d.z; D4[3] = d.w;
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const bool in = pos0 + pl0 + u < p.Lq;
                    L4[u] = in ? p.lse[li0 + u] : -INFINITY;
                    D4[u] = in ? p.Drow[li0 + u] : 0.f;
                }
            }
            // the mask rows' visibility bounds: key k0 + lane + 32 t sees
            // positions [lo[t], hi[t]] of the tile
            const bool masked = mask_mma && tile_masked(i);
            int lo[4], hi[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const long j = (long)k0 + lane + 32 * t, jrel = j - pos0 - off;
                long lo_l = max(jrel, 0L);
                const long hi_l = p.window > 0 ? jrel + p.window - 1 : (long)P - 1;
                if (j >= p.Lk) lo_l = P;
                lo[t] = (int)min(lo_l, (long)P);
                hi[t] = (int)max(-1L, min(hi_l, (long)P - 1));
            }
            if (lane == 0) {
                ok = mbar_wait(&qdo_empty[st], ((i >> 1) & 1u) ^ 1u, abort_flag, p.status, p.timeout_ns);
                if (ok) {
                    mbar_arrive_expect_tx(&qdo_full[st], 2 * kTile);
                    tma_load_4d(smem + kOffQ + st * kTile, &tmQ, 0, h0, pos0, b, &qdo_full[st]);
                    tma_load_4d(smem + kOffDO + st * kTile, &tmDO, 0, h0, pos0, b, &qdo_full[st]);
                    if (st) ++issued_qdo1; else ++issued_qdo0;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            // log2-domain lse (+inf for rows that do not exist or see nothing)
            // and D, scattered to columns pos * GP + head
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = (pl0 + u) * GP + hl;
                ld[(st * 2 + 0) * kM + c] = (L4[u] == -INFINITY) ? INFINITY : L4[u] * kLog2e;
                ld[(st * 2 + 1) * kM + c] = D4[u];
            }
            if (masked) {
                // the stage's mask rows (S^T two tiles back, their last reader,
                // completed before qdo_empty): 0 where the position sees the key
                uint8_t *ek = smem + kOffEK + st * kEBytes;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int r = lane + 32 * t;
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh) {
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int k = 8 * kh + 2 * u;
                            w[u] = ((k >= lo[t] && k <= hi[t]) ? 0u : 0xF180u) |
                                   ((k + 1 >= lo[t] && k + 1 <= hi[t]) ? 0u : 0xF180u) << 16;
                        }
                        *reinterpret_cast<uint4 *>(ek + (r >> 3) * 256 + kh * 128 + (r & 7) * 16) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            if (mask_mma) fence_proxy_async_smem();  // the tables are read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&qdo_full[st]);
        }
        if (lane == 0) {
            if (n_iter > 0) wait_noabort(kv_full, 0, p.status, p.timeout_ns);
            if (issued_qdo0) wait_noabort(&qdo_full[0], (issued_qdo0 - 1) & 1u, p.status, p.timeout_ns);
            if (issued_qdo1) wait_noabort(&qdo_full[1], (issued_qdo1 - 1) & 1u, p.status, p.timeout_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        // The whole warp runs this loop (so every operand is warp-uniform) and
        // one elected lane issues the MMAs and their commits.
        const uint32_t id_t = idesc_bf16_f32(kM, kM, 0, 0);       // S^T, dP^T: N = 128 q rows
        const uint32_t id_kv = idesc_bf16_f32(kM, kD, 1, 0);      // dV, dK: B MN-major
        const uint32_t id_q = idesc_bf16_f32(kM, kD, 1, 1);       // dQ: A and B MN-major
        const uint64_t d_k = smem_desc_sw128(smem_u32(smem + kOffK), 16, 1024);
        const uint64_t d_v = smem_desc_sw128(smem_u32(smem + kOffV), 16, 1024);
        const uint64_t d_q = smem_desc_sw128(smem_u32(smem + kOffQ), 16, 1024);
        const uint64_t d_do = smem_desc_sw128(smem_u32(smem + kOffDO), 16, 1024);
        const uint64_t d_ds = smem_desc_sw128(smem_u32(smem + kOffDS), kTile, 1024);
        const uint64_t d_kmn = smem_desc_sw128(smem_u32(smem + kOffK), kTile, 1024);
        auto wait_all = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status, p.timeout_ns));
        };
        const uint64_t d_ek = smem_desc_noswz(smem_u32(smem + kOffEK), 128, 256);
        const uint64_t d_eq = smem_desc_noswz(smem_u32(smem + kOffEQ), 128, 256);
        bool ok = n_iter > 0 && wait_all(kv_full, 0);
        // S^T(i) = K Q(i)^T into its own TMEM tile; issued for tile i+1 as
        // soon as the softmax-gradient threads have read S^T(i) out.
        auto issue_st = [&](int i) -> bool {
            const int st = i & 1;
            if (!wait_all(&qdo_full[st], (i >> 1) & 1u)) return false;
            if (i > 0 && !wait_all(s_consumed, (i - 1) & 1u)) return false;
            tc_fence_after();
            const uint64_t q_st = d_q + (uint64_t)((st * kTile) >> 4);
            const bool extra = mask_mma && tile_masked(i);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) mma_ss(tmem + kTmST, d_k + 2 * kk, q_st + 2 * kk, id_t, kk > 0);
                if (extra)  // + 0 / -2^100 where the position does not see the key
                    mma_ss(tmem + kTmST, d_ek + (uint64_t)((st * kEBytes) >> 4), d_eq, id_t, 1u);
                mma_commit(s_full);
            }
            __syncwarp();
            return true;
        };
        // dP^T(i) = V dO(i)^T; its columns held dS^T(i-1), read by dK(i-1),
        // which was issued before it (tcgen05 MMAs of one thread run in order)
        auto issue_dpt = [&](int i) {
            const uint64_t do_st = d_do + (uint64_t)(((i & 1) * kTile) >> 4);
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss(tmem + kTmDPT, d_v + 2 * kk, do_st + 2 * kk, id_t, kk > 0);
                mma_commit(dp_full);
            }
            __syncwarp();
        };
        if (ok) ok = issue_st(0);
        if (ok) issue_dpt(0);
        for (int i = 0; i < n_iter && ok; ++i) {
            const int st = i & 1;
            const uint64_t q_st = d_q + (uint64_t)((st * kTile) >> 4);
            const uint64_t do_st = d_do + (uint64_t)((st * kTile) >> 4);
            // scores of the next q tile, as soon as S^T(i) has been read
            if (i + 1 < n_iter && !issue_st(i + 1)) break;
            if (!wait_all(p_ready, i & 1u)) break;
            tc_fence_after();
            // dV += P^T dO and dK += dS^T Q: K = 128 q rows in steps of 16 (2048 bytes of the MN-major B)
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kM / 16; ++kk)
                    mma_ts(tmem + kTmDV, tmem + kTmPT + kk * 8, do_st + 128 * kk, id_kv, (i > 0 || kk > 0));
                mma_commit(pt_free);
#pragma unroll
                for (int kk = 0; kk < kM / 16; ++kk)
                    mma_ts(tmem + kTmDK, tmem + kTmDPT + kk * 8 + (kk >= kM / 32 ? kM / 4 : 0), q_st + 128 * kk,
                           id_kv, (i > 0 || kk > 0));
                mma_commit(&qdo_empty[st]);
            }
            __syncwarp();
            // dP^T of the next q tile ahead of dQ(i), which only the dQ epilogue waits for
            if (i + 1 < n_iter) {
                if (!wait_all(&qdo_full[(i + 1) & 1], ((i + 1) >> 1) & 1u)) break;
                issue_dpt(i + 1);
            }
            if (!wait_all(dq_free, (i & 1u) ^ 1u)) break;
            tc_fence_after();
            // dQ = dS K: K = 128 keys in steps of 16
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kM / 16; ++kk)
                    mma_ss(tmem + kTmDQ, d_ds + 128 * kk, d_kmn + 128 * kk, id_q, kk > 0);
                mma_commit(dq_full);
                mma_commit(ds_free);
            }
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(dkv_done);
            mma_commit(drain);
        }
        __syncwarp();
        wait_noabort(drain, 0, p.status, p.timeout_ns);
    } else if (warp <= 5 || warp >= 10) {
        // ------------------------------------------------------------ P and dS, one key row per warp pair
        constexpr int kCh = kM / 32;       // 16-column chunks per half
        const int quad = warp & 3;
        const int half = warp >= 10;       // q columns [64 half, 64 half + 64)
        const int c0 = half * kCh;
        const int r = quad * 32 + lane;
        const int j = k0 + r;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const float C = p.c_log2;
        bool ok = true;
        for (int i = 0; i < n_iter; ++i) {
            const int st = i & 1;
            int h0, pos0;
            iter_head(i, h0, pos0);
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&qdo_full[st], (i >> 1) & 1u, abort_flag, p.status, p.timeout_ns) &&
                                mbar_wait(s_full, i & 1u, abort_flag, p.status, p.timeout_ns))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // key j is visible to column c (position pos0 + c / GP) iff
            // pl = c / GP lies in [pl_lo, pl_hi]: j <= pos + off and, with a
            // window, j > pos + off - window (bounds exact in 64 bits, then
            // clamped to [-1, P])
            const long jrel = (long)j - pos0 - off;
            long lo_l = max(jrel, 0L);
            long hi_l = p.window > 0 ? jrel + p.window - 1 : (long)P - 1;
            if (j >= p.Lk) lo_l = P;  // keys past Lk see nothing
            const int pl_lo = (int)min(lo_l, (long)P);
            const int pl_hi = (int)max(-1L, min(hi_l, (long)P - 1));
            const bool need_mask = !mask_mma && __any_sync(0xffffffffu, pl_lo > 0 || pl_hi < P - 1);
            const float4 *l2v = reinterpret_cast<const float4 *>(ld + (st * 2 + 0) * kM);
            const float4 *ddv = reinterpret_cast<const float4 *>(ld + (st * 2 + 1) * kM);

            // phase 1: P = exp2(S C - lse2) from S^T, kept as bf16 pairs; then S^T is free
            // TMEM loads are pipelined one 16-column chunk ahead of the arithmetic.
            // Compiled twice: tiles with no masked element (most of them) run
            // without the per-element visibility test.
            uint32_t pk[kM / 4];
            // 16 columns of chunk c (0..kCh-1 within the half) from S^T values sr -> 8 bf16 pairs
            auto p_chunk = [&](auto masked_tag, const uint32_t *sr, int c, uint32_t *q) {
                constexpr bool kMasked = decltype(masked_tag)::value;
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 l4 = l2v[4 * (c0 + c) + e4];
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
                    float pe[4], xa[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) xa[u] = fmaf(__uint_as_float(sr[4 * e4 + u]), C, -lv[u]);
                    // on tiles with no masked element, one pair in eight on the FMA
                    // pipe (fast_exp2x2) to offload the MUFU unit (measured: 2.7 %
                    // faster on the dense layer; a quarter or a half were slower)
#pragma unroll
                    for (int u = 0; u < 4; u += 2) {
                        if (!kMasked && e4 == 3 && u == 2) {
                            const float2 f = fast_exp2x2(make_float2(xa[u], xa[u + 1]));
                            pe[u] = f.x;
                            pe[u + 1] = f.y;
                        } else {
                            pe[u] = ex2(xa[u]);
                            pe[u + 1] = ex2(xa[u + 1]);
                        }
                    }
                    if (kMasked) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int pl = (16 * (c0 + c) + 4 * e4 + u) / GP;
                            pe[u] = (pl >= pl_lo && pl <= pl_hi) ? pe[u] : 0.f;
                        }
                    }
                    q[2 * e4] = pack_bf16x2(pe[0], pe[1]);
                    q[2 * e4 + 1] = pack_bf16x2(pe[2], pe[3]);
                }
            };
            auto phase1 = [&](auto masked_tag) {
                uint32_t sbuf[2][16];
                tmem_ld16(trow + kTmST + 16 * c0, sbuf[0]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < kCh; ++c) {
                    if (c + 1 < kCh) tmem_ld16(trow + kTmST + 16 * (c0 + c + 1), sbuf[(c + 1) & 1]);
                    p_chunk(masked_tag, sbuf[c & 1], c, &pk[8 * c]);
                    tmem_wait_ld();
                }
            };
            if constexpr (mask_mma) {
                phase1(std::false_type{});
            } else {
                if (need_mask)
                    phase1(std::true_type{});
                else
                    phase1(std::false_type{});
            }
            // P^T into its columns once dV(i-1) has read the previous P^T
            if (i > 0 &&
                !__all_sync(0xffffffffu, mbar_wait(pt_free, (i - 1) & 1u, abort_flag, p.status, p.timeout_ns))) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < kCh / 2; ++c) tmem_st16(trow + kTmPT + kM / 4 * half + 16 * c, &pk[16 * c]);
            tc_fence_before();
            mbar_arrive(s_consumed);  // S^T(i+1) may be computed into these columns now

            // phase 2: dS = P (dP - D) from dP^T; dS^T (bf16 pairs) over the read
            // columns of dP^T, dS into shared memory (MN-major) for dQ
            if (!__all_sync(0xffffffffu, mbar_wait(dp_full, i & 1u, abort_flag, p.status, p.timeout_ns) &&
                                             (i == 0 || mbar_wait(ds_free, (i - 1) & 1u, abort_flag, p.status,
                                                                  p.timeout_ns)))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // chunk c: dS from dP^T values dr and P pairs pp; dS^T over 8 columns of
            // dP^T this warp has read (64 half + 8c .. + 7), dS into shared memory
            auto ds_chunk = [&](const uint32_t *dr, const uint32_t *pp, int c) {
                uint32_t dk[8];
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 d4 = ddv[4 * (c0 + c) + e4];
                    const __nv_bfloat162 p01 = *reinterpret_cast<const __nv_bfloat162 *>(&pp[2 * e4]);
                    const __nv_bfloat162 p23 = *reinterpret_cast<const __nv_bfloat162 *>(&pp[2 * e4 + 1]);
                    const float ds0 = __low2float(p01) * (__uint_as_float(dr[4 * e4 + 0]) - d4.x);
                    const float ds1 = __high2float(p01) * (__uint_as_float(dr[4 * e4 + 1]) - d4.y);
                    const float ds2 = __low2float(p23) * (__uint_as_float(dr[4 * e4 + 2]) - d4.z);
                    const float ds3 = __high2float(p23) * (__uint_as_float(dr[4 * e4 + 3]) - d4.w);
                    dk[2 * e4] = pack_bf16x2(ds0, ds1);
                    dk[2 * e4 + 1] = pack_bf16x2(ds2, ds3);
                }
                tmem_st8(trow + kTmDPT + 16 * c0 + 8 * c, dk);
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8) {
                    const int chunk = 2 * (c0 + c) + q8;  // 8-column chunk index 0..15
                    const int atom = chunk >> 3, cc = chunk & 7;
                    *reinterpret_cast<uint4 *>(smem + kOffDS + atom * kTile + r * 128 + ((cc ^ (r & 7)) << 4)) =
                        make_uint4(dk[4 * q8], dk[4 * q8 + 1], dk[4 * q8 + 2], dk[4 * q8 + 3]);
                }
            };
            uint32_t dbuf[2][16];
            tmem_ld16(trow + kTmDPT + 16 * c0, dbuf[0]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < kCh; ++c) {
                if (c + 1 < kCh) tmem_ld16(trow + kTmDPT + 16 * (c0 + c + 1), dbuf[(c + 1) & 1]);
                ds_chunk(dbuf[c & 1], &pk[8 * c], c);
                tmem_wait_ld();
            }
            tmem_wait_st();
            fence_proxy_async_smem();  // dS in shared memory is read by the tensor core next
            tc_fence_before();
            mbar_arrive(p_ready);
        }
        // ---- dK, dV of this key row, 16 columns at a time (32 per half)
        const bool done = ok && n_iter > 0 &&
                          __all_sync(0xffffffffu, mbar_wait(dkv_done, 0, abort_flag, p.status, p.timeout_ns));
        if (done) tc_fence_after();
        const bool write = (done || (n_iter == 0 && !*abort_flag)) && j < p.Lk;
        const size_t base = (((size_t)b * p.Lk + (j < p.Lk ? j : 0)) * p.Hkv + g) * kD;
#pragma unroll
        for (int cc = 0; cc < kD / 32; ++cc) {
            const int c = half * (kD / 32) + cc;
            uint32_t va[16], ka[16];
            if (done) {  // warp-uniform
                tmem_ld16(trow + kTmDV + 16 * c, va);
                tmem_ld16(trow + kTmDK + 16 * c, ka);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) va[e] = ka[e] = 0u;
            }
            if (write) {
                uint4 *dv4 = reinterpret_cast<uint4 *>(p.dv + base + 16 * c);
                uint4 *dk4 = reinterpret_cast<uint4 *>(p.dk + base + 16 * c);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint4 a, bb;
                    a.x = pack_bf16x2(__uint_as_float(va[8 * h + 0]), __uint_as_float(va[8 * h + 1]));
                    a.y = pack_bf16x2(__uint_as_float(va[8 * h + 2]), __uint_as_float(va[8 * h + 3]));
                    a.z = pack_bf16x2(__uint_as_float(va[8 * h + 4]), __uint_as_float(va[8 * h + 5]));
                    a.w = pack_bf16x2(__uint_as_float(va[8 * h + 6]), __uint_as_float(va[8 * h + 7]));
                    bb.x = pack_bf16x2(__uint_as_float(ka[8 * h + 0]) * p.scale, __uint_as_float(ka[8 * h + 1]) * p.scale);
                    bb.y = pack_bf16x2(__uint_as_float(ka[8 * h + 2]) * p.scale, __uint_as_float(ka[8 * h + 3]) * p.scale);
                    bb.z = pack_bf16x2(__uint_as_float(ka[8 * h + 4]) * p.scale, __uint_as_float(ka[8 * h + 5]) * p.scale);
                    bb.w = pack_bf16x2(__uint_as_float(ka[8 * h + 6]) * p.scale, __uint_as_float(ka[8 * h + 7]) * p.scale);
                    dv4[h] = a;
                    dk4[h] = bb;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ dQ: TMEM -> smem -> TMA reduce-add
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const bool issuer = (warp == 6 && lane == 0);
        grid_dep_wait();  // the pre-pass clears the accumulator
        float *stg = reinterpret_cast<float *>(smem + kOffStg);
        for (int i = 0; i < n_iter; ++i) {
            int h0, pos0;
            iter_head(i, h0, pos0);
            if (!__all_sync(0xffffffffu, mbar_wait(dq_full, i & 1u, abort_flag, p.status, p.timeout_ns)))
                break;
            tc_fence_after();
            uint32_t a[2][32];
            tmem_ld32(trow + kTmDQ, a[0]);
            tmem_ld32(trow + kTmDQ + 32, a[1]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(dq_free);
            if (!__all_sync(0xffffffffu, mbar_wait(stg_free, (i & 1u) ^ 1u, abort_flag, p.status, p.timeout_ns)))
                break;
            // columns 32 hh .. 32 hh + 31 of row `row` fill 128 bytes of half hh;
            // 16-byte chunk j lands at chunk j ^ (row & 7) (the TMA 128-byte
            // swizzle), so 8 consecutive rows hit 8 different bank groups
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float4 v;
                    v.x = __uint_as_float(a[hh][4 * j + 0]) * p.scale;
                    v.y = __uint_as_float(a[hh][4 * j + 1]) * p.scale;
                    v.z = __uint_as_float(a[hh][4 * j + 2]) * p.scale;
                    v.w = __uint_as_float(a[hh][4 * j + 3]) * p.scale;
                    *reinterpret_cast<float4 *>(reinterpret_cast<uint8_t *>(stg) + hh * (kM * 128) + row * 128 +
                                                ((j ^ (row & 7)) << 4)) = v;
                }
            fence_proxy_async_smem();
            mbar_arrive(stg_full);
            if (issuer) {
                if (!mbar_wait(stg_full, i & 1u, abort_flag, p.status, p.timeout_ns)) break;
                // the accumulator's lines stay in L2 ahead of the streamed q and
                // dO tiles, for the other key tiles' adds and the final
                // conversion (window-128 backward 135 -> 132 us at B1 L4096)
                const uint64_t pol = l2_policy_evict_last();
                tma_reduce_add_4d_hint(&tmDQ, stg, 0, h0, pos0, b, pol);
                tma_reduce_add_4d_hint(&tmDQ, reinterpret_cast<uint8_t *>(stg) + kM * 128, kD / 2, h0, pos0, b, pol);
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(stg_free);
            }
        }
        if (issuer) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// The backward's last step, one launch: blocks [0, n_conv) turn the fp32 dQ
// accumulator into bf16 (8 values per thread); block n_conv + h sums head h's
// B * Lq dsink terms in a fixed order (deterministic).
__global__ void __launch_bounds__(256) bwd_finish_kernel(const float *__restrict__ acc, __nv_bfloat16 *__restrict__ dq,
                                                         size_t n8, unsigned n_conv, const float *__restrict__ terms,
                                                         float *__restrict__ dsinks, long nterms)
{
    grid_dep_wait();  // launched ahead of the main kernel's end: its dQ and the pre-pass's terms
    if (blockIdx.x >= n_conv) {
        __shared__ float red[256];
        const int h = (int)(blockIdx.x - n_conv), t = threadIdx.x;
        const float *row = terms + (size_t)h * nterms;
        float sum = 0.f;
        for (long e = t; e < nterms; e += 256) sum += row[e];
        red[t] = sum;
        __syncthreads();
        for (int w = 128; w > 0; w >>= 1) {
            if (t < w) red[t] += red[t + w];
            __syncthreads();
        }
        if (t == 0) dsinks[h] = red[0];
        return;
    }
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const float4 v0 = reinterpret_cast<const float4 *>(acc)[2 * i];
    const float4 v1 = reinterpret_cast<const float4 *>(acc)[2 * i + 1];
    uint4 o;
    o.x = pack_bf16x2(v0.x, v0.y);
    o.y = pack_bf16x2(v0.z, v0.w);
    o.z = pack_bf16x2(v1.x, v1.y);
    o.w = pack_bf16x2(v1.z, v1.w);
    reinterpret_cast<uint4 *>(dq)[i] = o;
}

template <int GP>
cudaError_t launch_gp(const CUtensorMap &mq, const CUtensorMap &mdo, const CUtensorMap &mk, const CUtensorMap &mv,
                      const CUtensorMap &mdq, const BwdParams &p, dim3 grid, cudaStream_t st)
{
    cudaError_t e = cudaFuncSetAttribute(bwd_tc_kernel<GP>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, bwd_tc_kernel<GP>, mq, mdo, mk, mv, mdq, p);
}

}  // namespace

size_t bwd_tc_dq_acc_bytes(const AttnShape &s) { return (size_t)s.B * s.Lq * s.Hq * s.D * sizeof(float); }

cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const void *dout, const float *lse,
                          const float *Drow, const float *terms, float *dsinks, float *dq_acc, void *dq, void *dk,
                          void *dv, const AttnShape &s, cudaStream_t st)
{
    BwdParams p;
    p.B = s.B;
    p.Lq = s.Lq;
    p.Lk = s.Lk;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.window = s.window;
    p.G = s.Hq / s.Hkv;
    // query heads per q tile: the largest power of two up to 16 dividing G;
    // with 8 or more the mask is an MMA step whose -2^100 times
    // scale * log2(e) must stay far below any exponent, so a smaller scale
    // takes 4 (the per-element mask)
    const int gp_max = s.scale >= 0x1p-60f ? 16 : 4;
    int gp = 1;
    while (gp * 2 <= gp_max && p.G % (gp * 2) == 0) gp *= 2;
    p.P = kM / gp;
    p.n_htiles = p.G / gp;
    p.c_log2 = s.scale * kLog2e;
    p.scale = s.scale;
    p.lse = lse;
    p.Drow = Drow;
    p.dk = static_cast<__nv_bfloat16 *>(dk);
    p.dv = static_cast<__nv_bfloat16 *>(dv);
    p.status = device_status_ptr();
    p.timeout_ns = wait_timeout_ns();

    alignas(64) CUtensorMap mq, mdo, mk, mv, mdq;
    const uint64_t qd[4] = {(uint64_t)kD, (uint64_t)s.Hq, (uint64_t)s.Lq, (uint64_t)s.B};
    const uint64_t qs2[3] = {(uint64_t)kD * 2, (uint64_t)s.Hq * kD * 2, (uint64_t)s.Lq * s.Hq * kD * 2};
    const uint64_t qs4[3] = {(uint64_t)kD * 4, (uint64_t)s.Hq * kD * 4, (uint64_t)s.Lq * s.Hq * kD * 4};
    const uint32_t qbox[4] = {(uint32_t)kD, (uint32_t)gp, (uint32_t)p.P, 1u};
    const uint32_t dqbox[4] = {(uint32_t)kD / 2, (uint32_t)gp, (uint32_t)p.P, 1u};  // 128-byte fp32 rows
    const uint64_t kd[4] = {(uint64_t)kD, (uint64_t)s.Hkv, (uint64_t)s.Lk, (uint64_t)s.B};
    const uint64_t ks2[3] = {(uint64_t)kD * 2, (uint64_t)s.Hkv * kD * 2, (uint64_t)s.Lk * s.Hkv * kD * 2};
    const uint32_t kbox[4] = {(uint32_t)kD, 1u, (uint32_t)kM, 1u};
    if (!encode_tensor_map_4d(&mq, const_cast<void *>(q), 2, qd, qs2, qbox, true) ||
        !encode_tensor_map_4d(&mdo, const_cast<void *>(dout), 2, qd, qs2, qbox, true) ||
        !encode_tensor_map_4d(&mk, const_cast<void *>(k), 2, kd, ks2, kbox, true) ||
        !encode_tensor_map_4d(&mv, const_cast<void *>(v), 2, kd, ks2, kbox, true) ||
        !encode_tensor_map_4d(&mdq, dq_acc, 4, qd, qs4, dqbox, true))
        return cudaErrorInvalidValue;
    // dq_acc arrives zeroed (the row pre-pass clears it)
    cudaError_t e;
    const long long n_cta = (long long)((s.Lk + kM - 1) / kM) * s.Hkv * s.B;
    if (n_cta > 0x7fffffffLL) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)n_cta);
    switch (gp) {
    case 1: e = launch_gp<1>(mq, mdo, mk, mv, mdq, p, grid, st); break;
    case 2: e = launch_gp<2>(mq, mdo, mk, mv, mdq, p, grid, st); break;
    case 4: e = launch_gp<4>(mq, mdo, mk, mv, mdq, p, grid, st); break;
    case 8: e = launch_gp<8>(mq, mdo, mk, mv, mdq, p, grid, st); break;
    default: e = launch_gp<16>(mq, mdo, mk, mv, mdq, p, grid, st); break;
    }
    if (e != cudaSuccess) return e;
    const size_t n8 = (size_t)s.B * s.Lq * s.Hq * s.D / 8;
    const size_t n_conv = (n8 + 255) / 256;
    if (n_conv + s.Hq > 0x7fffffffu) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n_conv + s.Hq));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, bwd_finish_kernel, (const float *)dq_acc, static_cast<__nv_bfloat16 *>(dq), n8,
                              (unsigned)n_conv, terms, dsinks, (long)s.B * s.Lq);
}

bool bwd_tc_supported(const AttnShape &s)
{
    return s.D == kD && s.Hq % s.Hkv == 0 && s.B <= 65535 && s.Hkv <= 65535;
}

}  // namespace attn_sink
