// fwd_band.cu -- bf16 prefill forward of sink-softmax GQA attention for
// causal layers banded to a short window (gpt-oss alternates dense layers
// with layers banded to sliding_window = 128: "GPT-OSS 20B Egitimi: Unsloth,
// A100 ve Hopper Uyumlulugu", section 1; "GPT-OSS-120B 4-bit ...", section 3).
//
// What it computes ("GPT-OSS on day 0", section "Sink Attention"): for each
// query row, the softmax over its visible keys and the head's sink logit,
// O = sum_j p_j v_j and the log-sum-exp including the sink.
//
// Design (B200).  A work item is 128 query rows = P positions x Gp query heads
// of one KV group (GQA packing, as in the dense forward).  The rows of an item
// see keys [pos0 + off - W + 1, pos0 + off + P - 1]: W + P - 1 keys, 143 for
// W = 128 and P = 16.  So one K/V tile of KN >= W + P - 1 rows (144) holds
// every key of the item, and the item is ONE score MMA (M = 128, N = KN), one
// exact softmax (no running maximum, no rescale), and one P.V MMA.
//  * One CTA per SM (all 512 TMEM columns), two softmax warpgroups that take
//    alternate items, so one item's softmax overlaps the other's MMAs, loads
//    and epilogue.  The grid has one CTA per item; running CTAs take over the
//    items of CTAs that have not started through cluster launch control.
//  * Warp 0: TMA producer.  Q (16 KB) and the K and V tiles (KN x 128 B each,
//    starting at a negative row where the band reaches before key 0: the TMA
//    fills rows outside the tensor with zeros) in four stages, so items ahead
//    of the two being computed are in flight.
//  * Warp 1: the MMA issue loop (whole warp, one elected lane issuing),
//    polling the barriers of both warpgroups' items and issuing whichever
//    product is ready: P.V of item r as soon as its P is written, S = Q K^T
//    of item r + 2 into the same TMEM half once P.V(r) is issued (the tensor
//    pipe runs them in order) and its Q, K have landed.
//  * Warps 4-7 and 8-11 (registers moved to them from warpgroup 0 with
//    setmaxnreg), one thread per row: the whole score row (KN columns)
//    comes out of TMEM in one go into registers; masks only on the 16-column
//    chunks where some row of the warp needs them; m = max(sink, row max);
//    P = exp2(S C - m) as bf16 over S; l.  Epilogue: O / l written into the
//    item's K buffer (its Q buffer for narrow bands; either is dead once S is
//    done) in the 128-byte-swizzled layout of an output box, and stored with
//    one TMA tensor store (a box that would run into the next packed sequence
//    is stored row by row instead); lse row by row.  The buffer goes back to
//    the producer once the store has read it, which the storing thread checks
//    in the warpgroup's next item rather than waiting for it right away.
//  * Every wait is bounded; on expiry the CTA raises a status bit, waits
//    (bounded) for its own TMA loads, stores and MMAs, frees tensor memory and
//    exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

constexpr int kM = 128;
constexpr int kD = 64;
constexpr int kThreads = 384;  // warpgroup 0: producer, MMA (2 warps idle); warpgroups 1, 2: softmax
// Registers: launched at 168 per thread (384 threads, one CTA per SM); warpgroup
// 0 then gives up all but 56 and the softmax warpgroups take 224 each, so the
// score row of a thread stays in registers: 128 x 56 + 256 x 224 = 384 x 168.
// (Each SM sub-partition holds one warp of every warpgroup: 56 + 2 x 224 fits
// its 16K registers as 3 x 168 does.)
constexpr int kRegsLaunch = 168, kRegsCtl = 56, kRegsSoftmax = 224;
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr int kNS = 4;         // Q/K/V stages
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kTmemCols = 512;  // warpgroup w: S at [256 w, 256 w + KN), O at [256 w + 192, 256 w + 256)
constexpr int kTmO = 192;

template <int KN>
struct BandCfg {
    static_assert(KN % 16 == 0 && KN >= 16 && KN <= 144, "KN: a multiple of 16 up to 144");
    static constexpr int kQBytes = kM * kD * 2;
    static constexpr int kKVBytes = KN * kD * 2;
    static constexpr int kOffQ = 0;                       // [kNS]
    static constexpr int kOffK = kNS * kQBytes;           // [kNS]
    static constexpr int kOffV = kOffK + kNS * kKVBytes;  // [kNS]
    // The band's staircase mask as one more K = 16 step of the score MMA:
    // S += E_q E_k^T with E_q[row][k] = (k == the row's position in the item)
    // and E_k[col][k] = -2^100 where key col is outside position k's window,
    // else 0 (bf16, K-major without swizzle: 8-row groups of 256 bytes).
    static constexpr int kOffEq = kOffV + kNS * kKVBytes;  // 128 rows x 32 bytes
    static constexpr int kOffEk = kOffEq + kM * 32;        // KN rows x 32 bytes
    static constexpr int kOffBar = kOffEk + KN * 32;
    // The item's O is staged in its K buffer when that holds 16 KB (K is dead
    // once S is done and is only needed again two items of this warpgroup
    // later), else in its Q buffer.
    static constexpr bool kStageInK = kKVBytes >= kQBytes;
    // q_full q_empty k_full k_empty v_full v_empty [kNS each]; s_full p_full o_done o_free stg_ready [2 each];
    // drain; item_full[4] item_empty[4]; clc[kClcDepth]
    static constexpr int kNumBar = 6 * kNS + 10 + 1 + 8 + kClcDepth;
    static constexpr int kOffMisc = (kOffBar + kNumBar * 8 + 15) / 16 * 16;
    // tmem slot (+0), abort flag (+4), item ring (+16), launch-control responses (+32, 16 bytes each)
    static_assert(32 + 16 * kClcDepth <= 128, "misc area");
    static constexpr int kSmemUsed = kOffMisc + 128 + 1024;  // + slack for 1024-byte alignment
    // more than half the SM's shared memory even for narrow bands: a second
    // CTA on the SM would only wait for the first one's tensor memory
    static constexpr int kSmemBytes = kSmemUsed < 116 * 1024 ? 116 * 1024 : kSmemUsed;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct BandParams {
    int B, Lq, Lk, Hq, Hkv, window;
    const int *cu_q, *cu_k;  // packed ragged sequences (else nullptr)
    int total_q, total_k;
    long long lse_hs;        // lse stride between heads: Lq, or total_q for packed sequences
    int G, Gp, P;
    int n_ptiles, n_htiles, n_items;
    int mask_mma;  // P <= 16: the staircase mask comes from the extra MMA step
    float c_log2;  // scale * log2(e)
    const float *sinks;
    __nv_bfloat16 *out;
    float *lse;
    unsigned *status;
    long long timeout_ns;
};

struct BandItem {
    int pos0, h0, b, js;   // first position, first head, batch, first key of the K/V tile (in the sequence)
    int Lq, Lk;            // the sequence's query and key counts
    int qrow0, krow0, tb;  // tensor-map rows of its position 0 / key 0, outer coordinate
    long long orow0;       // output row of its position 0
    long long lrow0;       // lse index of (head 0, position 0)
    bool empty;            // past the end of a shorter packed sequence
};

// Item i: head tiles fastest, then position tiles, then batches, so the CTAs
// running at once cover neighbouring positions of every KV group and share
// K/V rows through L2.
__device__ __forceinline__ BandItem band_item(const BandParams &p, int i)
{
    BandItem it;
    it.h0 = (i % p.n_htiles) * p.Gp;
    const int r = i / p.n_htiles;
    it.pos0 = (r % p.n_ptiles) * p.P;
    it.b = r / p.n_ptiles;
    const SeqRows sq = seq_rows(p.cu_q, it.b, p.Lq, p.total_q);
    const SeqRows sk = seq_rows(p.cu_k, it.b, p.Lk, p.total_k);
    it.Lq = sq.len;
    it.Lk = sk.len;
    it.qrow0 = sq.row0;
    it.krow0 = sk.row0;
    it.tb = p.cu_q ? 0 : it.b;
    it.orow0 = p.cu_q ? (long long)sq.row0 : (long long)it.b * p.Lq;
    it.lrow0 = p.cu_q ? (long long)sq.row0 : (long long)it.b * p.Hq * p.Lq;
    it.empty = it.pos0 >= it.Lq;
    it.js = it.pos0 + (it.Lk - it.Lq) - p.window + 1;
    return it;
}

__device__ __forceinline__ bool wait_noabort(uint64_t *bar, uint32_t parity, unsigned *status, long long tmo)
{
    int never = 0;
    return mbar_wait<false>(bar, parity, &never, status, tmo > 1000000000LL ? tmo : 1000000000LL);
}

template <int KN>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_band_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const BandParams p)
{
    using Cfg = BandCfg<KN>;
    constexpr int kChunks = KN / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *q_full = bars, *q_empty = bars + kNS;
    uint64_t *k_full = bars + 2 * kNS, *k_empty = bars + 3 * kNS;
    uint64_t *v_full = bars + 4 * kNS, *v_empty = bars + 5 * kNS;
    uint64_t *s_full = bars + 6 * kNS;  // [2]: one per warpgroup
    uint64_t *p_full = s_full + 2;      // [2]
    uint64_t *o_done = p_full + 2;      // [2]
    uint64_t *o_free = o_done + 2;      // [2]
    uint64_t *stg_ready = o_free + 2;   // [2]: every row of the item staged for its tensor store
    uint64_t *drain = stg_ready + 2;
    uint64_t *item_full = drain + 1, *item_empty = item_full + 4;
    uint64_t *clc_bar = item_empty + 4;  // [kClcDepth]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Cfg::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffMisc + 4);
    volatile int *ring = reinterpret_cast<volatile int *>(smem + Cfg::kOffMisc + 16);
    uint8_t *clc_resp = smem + Cfg::kOffMisc + 32;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);  // S, or the epilogue once the O store has read the buffer
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(&s_full[w], 1);
            mbar_init(&p_full[w], 128);
            mbar_init(&o_done[w], 1);
            mbar_init(&o_free[w], 128);
            mbar_init(&stg_ready[w], 128);
        }
        mbar_init(drain, 1);
        for (int r = 0; r < 4; ++r) {
            mbar_init(&item_full[r], 1);
            mbar_init(&item_empty[r], 5);  // the MMA warp and the four warps of the item's warpgroup
        }
        for (int d = 0; d < kClcDepth; ++d) mbar_init(&clc_bar[d], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (p.mask_mma) {
        // E_q and E_k of the mask step, element (row, k) at byte
        // (row / 8) 256 + (k / 8) 128 + (row % 8) 16 + (k % 8) 2
        uint16_t *eq = reinterpret_cast<uint16_t *>(smem + Cfg::kOffEq);
        uint16_t *ek = reinterpret_cast<uint16_t *>(smem + Cfg::kOffEk);
        constexpr uint16_t kOne = 0x3F80u, kBig = 0xF180u;  // bf16 1 and -2^100
        for (int i = threadIdx.x; i < (kM + KN) * 16; i += kThreads) {
            const bool isq = i < kM * 16;
            const int j = isq ? i : i - kM * 16;
            const int row = j >> 4, k = j & 15;
            const uint16_t v = isq ? ((k == row / p.Gp) ? kOne : (uint16_t)0)
                                   : ((k < p.P && (row < k || row > k + p.window - 1)) ? kBig : (uint16_t)0);
            (isq ? eq : ek)[((row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2) >> 1] = v;
        }
        fence_proxy_async_smem();  // read by the tensor core
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // r-th item of this CTA: its own (blockIdx.x), then those of the CTAs whose
    // launch it cancels (kClcDepth requests kept in flight); published in a
    // 4-slot ring, and -1 twice at the end (once for each warpgroup).  Items
    // past the end of a shorter packed sequence are passed over here.
    ClcQueue<kClcDepth, false> clc{clc_bar, clc_resp};
    auto publish = [&](int r, int w) -> bool {
        const int sl = r & 3;
        if (!mbar_wait<false>(&item_empty[sl], ((r >> 2) & 1u) ^ 1u, abort_flag, p.status, p.timeout_ns)) return false;
        ring[sl] = w;
        mbar_arrive(&item_full[sl]);
        return true;
    };
    auto producer_item = [&](int r) -> int {
        int w = r == 0 ? (int)blockIdx.x : clc.next(abort_flag, p.status, p.timeout_ns);
        clc.fill();  // keep kClcDepth requests in flight
        while (w >= 0 && band_item(p, w).empty) {
            w = clc.next(abort_flag, p.status, p.timeout_ns);
            clc.fill();
        }
        if (clc.failed) return -1;
        if (!publish(r, w)) return -1;
        if (w < 0) publish(r + 1, -1);
        return w;
    };
    auto consumer_item = [&](int r) -> int {
        const int sl = r & 3;
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&item_full[sl], (r >> 2) & 1u, abort_flag, p.status, p.timeout_ns)))
            return -1;
        const int w = ring[sl];
        __syncwarp();
        if (lane == 0) mbar_arrive(&item_empty[sl]);
        return w;
    };

    if (warp < 4) {
    regs_release<kRegsCtl>();  // the whole warpgroup; warps 2 and 3 have no role
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmO);
            uint32_t nq = 0, nk = 0, nv = 0;  // loads issued (the stage of load n is n % kNS)
            int r = 0;
            for (int w = producer_item(0); w >= 0; w = producer_item(++r)) {
                const BandItem t = band_item(p, w);
                const int st = r % kNS;
                const uint32_t ph = ((r / kNS) & 1u) ^ 1u;
                const int g = t.h0 / p.G;
                if (!mbar_wait<false>(&q_empty[st], ph, abort_flag, p.status, p.timeout_ns)) break;
                mbar_arrive_expect_tx(&q_full[st], Cfg::kQBytes);
                tma_load_4d(smem + Cfg::kOffQ + st * Cfg::kQBytes, &tmQ, 0, t.h0, t.qrow0 + t.pos0, t.tb,
                            &q_full[st]);
                ++nq;
                if (!mbar_wait<false>(&k_empty[st], ph, abort_flag, p.status, p.timeout_ns)) break;
                mbar_arrive_expect_tx(&k_full[st], Cfg::kKVBytes);
                tma_load_4d(smem + Cfg::kOffK + st * Cfg::kKVBytes, &tmK, 0, g, t.krow0 + t.js, t.tb, &k_full[st]);
                ++nk;
                if (!mbar_wait<false>(&v_empty[st], ph, abort_flag, p.status, p.timeout_ns)) break;
                mbar_arrive_expect_tx(&v_full[st], Cfg::kKVBytes);
                tma_load_4d(smem + Cfg::kOffV + st * Cfg::kKVBytes, &tmV, 0, g, t.krow0 + t.js, t.tb, &v_full[st]);
                ++nv;
            }
            // every load issued, and a launch-control request in flight, lands before the CTA exits
            clc.drain(p.status, p.timeout_ns);
            for (uint32_t n = nq > kNS ? nq - kNS : 0; n < nq; ++n)
                wait_noabort(&q_full[n % kNS], (n / kNS) & 1u, p.status, p.timeout_ns);
            for (uint32_t n = nk > kNS ? nk - kNS : 0; n < nk; ++n)
                wait_noabort(&k_full[n % kNS], (n / kNS) & 1u, p.status, p.timeout_ns);
            for (uint32_t n = nv > kNS ? nv - kNS : 0; n < nv; ++n)
                wait_noabort(&v_full[n % kNS], (n / kNS) & 1u, p.status, p.timeout_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t id_s = idesc_bf16_f32(kM, KN, 0);
        const uint32_t id_pv = idesc_bf16_f32(kM, kD, 1);
        const uint64_t eq_desc = smem_desc_noswz(smem_u32(smem + Cfg::kOffEq), 128, 256);
        const uint64_t ek_desc = smem_desc_noswz(smem_u32(smem + Cfg::kOffEk), 128, 256);
        // every lane has seen the phase complete (a lane that has not yet is retried later)
        auto ready = [&](uint64_t *bar, uint32_t parity) { return __all_sync(0xffffffffu, mbar_test(bar, parity)); };
        // S = Q K^T of item r into its warpgroup's TMEM half
        auto issue_s = [&](int r) {
            const int st = r % kNS;
            tc_fence_after();
            const uint32_t qa = smem_u32(smem + Cfg::kOffQ + st * Cfg::kQBytes);
            const uint32_t kb = smem_u32(smem + Cfg::kOffK + st * Cfg::kKVBytes);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_ss(tmem + 256 * (r & 1), smem_desc_sw128(qa + kk * 32, 16, 1024),
                           smem_desc_sw128(kb + kk * 32, 16, 1024), id_s, kk > 0 ? 1u : 0u);
                if (p.mask_mma) mma_ss(tmem + 256 * (r & 1), eq_desc, ek_desc, id_s, 1u);  // + the band's mask
                mma_commit(&s_full[r & 1]);
                mma_commit(Cfg::kStageInK ? &q_empty[st] : &k_empty[st]);  // the other one stages O
            }
            __syncwarp();
        };
        // O = P V of item r
        auto issue_pv = [&](int r) {
            const int st = r % kNS, wg = r & 1;
            tc_fence_after();
            const uint32_t vb = smem_u32(smem + Cfg::kOffV + st * Cfg::kKVBytes);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kChunks; ++kk)
                    mma_ts(tmem + 256 * wg + kTmO, tmem + 256 * wg + kk * 8,
                           smem_desc_sw128(vb + kk * 2048, KN * 128, 1024), id_pv, kk > 0 ? 1u : 0u);
                mma_commit(&o_done[wg]);
                mma_commit(&v_empty[st]);
            }
            __syncwarp();
        };
        // Out-of-order issue between the two warpgroups' streams, so that a
        // product whose operands are ready never waits behind one whose loads
        // are still in flight:
        //  * P.V of item r once S(r) is issued, P(r) written, V(r) landed and
        //    the warpgroup's previous epilogue has read its O;
        //  * S of item r once its warpgroup's TMEM half is free (P.V(r - 2)
        //    issued: the tensor pipe runs one thread's MMAs in order) and Q(r),
        //    K(r) have landed.
        // Items come from the ring without blocking; the loop polls, and gives
        // up (abort flag, status bit) after the wait limit without progress.
        int n_valid = 0, next_s = 0, next_pv = 0;
        bool end = false;
        uint64_t t_last = globaltimer_ns();
        while (true) {
            bool progress = false;
            if (!end && n_valid < next_pv + 3) {
                const int sl = n_valid & 3;
                if (ready(&item_full[sl], (n_valid >> 2) & 1u)) {
                    const int w = ring[sl];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&item_empty[sl]);
                    if (w < 0)
                        end = true;
                    else
                        ++n_valid;
                    progress = true;
                }
            }
            if (next_pv < next_s) {
                const int r = next_pv, wg = r & 1;
                if (ready(&p_full[wg], (r >> 1) & 1u) && ready(&v_full[r % kNS], (r / kNS) & 1u) &&
                    ready(&o_free[wg], ((r >> 1) & 1u) ^ 1u)) {
                    issue_pv(r);
                    ++next_pv;
                    progress = true;
                }
            }
            if (next_s < n_valid && next_s < next_pv + 2) {
                const int r = next_s;
                const uint32_t ph = (r / kNS) & 1u;
                if (ready(&q_full[r % kNS], ph) && ready(&k_full[r % kNS], ph)) {
                    issue_s(r);
                    ++next_s;
                    progress = true;
                }
            }
            if (end && next_pv == n_valid) break;
            const uint64_t now = globaltimer_ns();
            if (progress) {
                t_last = now;
            } else {
                if (*abort_flag) break;
                if ((long long)(now - t_last) > p.timeout_ns) {
                    if (lane == 0) {
                        *abort_flag = 1;
                        atomicOr(p.status, STATUS_TIMEOUT);
                    }
                    __syncwarp();
                    break;
                }
            }
        }
        if (elect_one()) mma_commit(drain);
        __syncwarp();
        wait_noabort(drain, 0, p.status, p.timeout_ns);
    }
    } else {
        regs_claim<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax + epilogue
        const int wg = (warp - 4) >> 2;  // softmax warpgroup: items r with r % 2 == wg
        const int quad = warp & 3;       // TMEM lane quadrant of this warp
        const int row = quad * 32 + lane;
        const uint32_t trow = tmem + 256 * wg + ((uint32_t)(quad * 32) << 16);
        const float C = p.c_log2;
        const bool storer = (warp == 4 + 4 * wg) && lane == 0;  // issues the warpgroup's tensor stores
        bool stores_issued = false;
        // The buffer an item's O was staged in is released once its tensor
        // store has read it; the storer checks that only in the next item's
        // pass, after that item's scores are in registers, instead of waiting
        // for the read right after the store.  The next item of the warpgroup
        // uses another stage, so its own loads never wait for that release.
        static_assert(kNS > 2, "a warpgroup's consecutive items in different stages");
        uint64_t *store_free = nullptr;
        for (int r = wg;; r += 2) {
            const int w = consumer_item(r);
            if (w < 0) break;
            const BandItem t = band_item(p, w);
            const int st = r % kNS;
            const int dp = row / p.Gp;
            const int pos = t.pos0 + dp;
            const int h = t.h0 + row % p.Gp;
            const bool row_valid = pos < t.Lq;
            const float sink2 = p.sinks[h] * kLog2e;
            // columns c of the tile (key js + c) this row sees: c in [c_lo, c_hi]
            const int c_lo = max(dp, -t.js);
            const int c_hi = row_valid ? min(dp + p.window - 1, t.Lk - 1 - t.js) : -1;
            // an item whose every row is valid and whose band lies inside the
            // sequence is masked by the MMA step alone (same for the whole item)
            const bool interior = p.mask_mma && t.js >= 0 && t.pos0 + p.P <= t.Lq && t.Lk - t.js >= p.P + p.window - 1;
            if (!__all_sync(0xffffffffu, mbar_wait<false>(&s_full[wg], (r >> 1) & 1u, abort_flag, p.status, p.timeout_ns)))
                break;
            tc_fence_after();

            // ---- masks of items at the edges of a sequence (or with more than 16
            // positions): masked scores become -inf in tensor memory, chunk by
            // chunk in a rolled loop, only where some row of the warp needs it;
            // the other items are masked by the MMA step, so the unrolled path
            // below carries no mask code
            if (!interior) {
#pragma unroll 1
                for (int c = 0; c < kChunks; ++c) {
                    if (!__any_sync(0xffffffffu, 16 * c < c_lo || 16 * c + 15 > c_hi)) continue;
                    uint32_t v[16];
                    tmem_ld16(trow + 16 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (16 * c + e < c_lo || 16 * c + e > c_hi) v[e] = __float_as_uint(-INFINITY);
                    tmem_st16(trow + 16 * c, v);
                }
                tmem_wait_st();
            }

            // ---- the score row, all KN columns, in one TMEM read
            uint32_t sr[kChunks][16];
#pragma unroll
            for (int c = 0; c < kChunks; ++c) tmem_ld16(trow + 16 * c, sr[c]);
            tmem_wait_ld();
            if (storer && store_free != nullptr) {
                bulk_wait_read_all();
                mbar_arrive(store_free);
                store_free = nullptr;
            }
            float mx[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mx[k] = fmax3(mx[k], __uint_as_float(sr[c][k]), __uint_as_float(sr[c][8 + k]));
            const float tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
            const float m = fmaxf(sink2, tmax * C);  // reference maximum, log2 units
            const float neg_m = (m == -INFINITY) ? 0.f : -m;
            float l = (sink2 == -INFINITY) ? 0.f : ex2(sink2 + neg_m);  // the sink's mass
            {
                // P = exp2(S C - m) as bf16 over the first KN/2 columns of S, and its row sum
                // (masked columns hold -inf: exp2 gives exactly 0 there)
                const float2 C2 = make_float2(C, C), M2 = make_float2(neg_m, neg_m);
                float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    uint32_t pk[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float2 x = ffma2(make_float2(__uint_as_float(sr[c][2 * e]),
                                                           __uint_as_float(sr[c][2 * e + 1])),
                                               C2, M2);
                        const float2 pe = make_float2(ex2(x.x), ex2(x.y));
                        acc[e & 1] = fadd2(acc[e & 1], pe);
                        pk[e] = pack_bf16x2(pe.x, pe.y);
                    }
                    tmem_st8(trow + 8 * c, pk);
                }
                l += (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[wg]);

            // ---- epilogue: O / l into the item's Q buffer, one tensor store
            if (!__all_sync(0xffffffffu, mbar_wait<false>(&o_done[wg], (r >> 1) & 1u, abort_flag, p.status, p.timeout_ns)))
                break;
            tc_fence_after();
            uint32_t o[2][32];
            tmem_ld32(trow + kTmO, o[0]);
            tmem_ld32(trow + kTmO + 32, o[1]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&o_free[wg]);
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4 ov[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                ov[c].x = pack_bf16x2(__uint_as_float(o[c / 4][(c % 4) * 8 + 0]) * inv,
                                      __uint_as_float(o[c / 4][(c % 4) * 8 + 1]) * inv);
                ov[c].y = pack_bf16x2(__uint_as_float(o[c / 4][(c % 4) * 8 + 2]) * inv,
                                      __uint_as_float(o[c / 4][(c % 4) * 8 + 3]) * inv);
                ov[c].z = pack_bf16x2(__uint_as_float(o[c / 4][(c % 4) * 8 + 4]) * inv,
                                      __uint_as_float(o[c / 4][(c % 4) * 8 + 5]) * inv);
                ov[c].w = pack_bf16x2(__uint_as_float(o[c / 4][(c % 4) * 8 + 6]) * inv,
                                      __uint_as_float(o[c / 4][(c % 4) * 8 + 7]) * inv);
            }
            if (row_valid)
                p.lse[(size_t)(t.lrow0 + (long long)h * p.lse_hs + pos)] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
            // A box that would run past the end of a packed sequence (into the
            // next one) is written row by row; otherwise one tensor store, whose
            // box the TMA clips at the end of a fixed-length sequence.  The
            // storing thread waits (bounded) until all 128 rows are staged.
            uint8_t *stg = Cfg::kStageInK ? smem + Cfg::kOffK + st * Cfg::kKVBytes : smem + Cfg::kOffQ + st * Cfg::kQBytes;
            uint64_t *stg_free = Cfg::kStageInK ? &k_empty[st] : &q_empty[st];
            const bool ragged = p.cu_q != nullptr && t.pos0 + p.P > t.Lq;
            if (ragged) {
                if (row_valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((size_t)(t.orow0 + pos) * p.Hq + h) * kD);
#pragma unroll
                    for (int c = 0; c < 8; ++c) dst[c] = ov[c];
                }
            } else {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(stg + row * 128 + ((c ^ (row & 7)) << 4)) = ov[c];
                fence_proxy_async_smem();
            }
            mbar_arrive(&stg_ready[wg]);
            if (storer) {
                if (!mbar_wait<false>(&stg_ready[wg], (r >> 1) & 1u, abort_flag, p.status, p.timeout_ns)) break;
                if (!ragged) {
                    tma_store_4d(&tmO, stg, 0, t.h0, t.qrow0 + t.pos0, t.tb);
                    bulk_commit_group();
                    stores_issued = true;
                    store_free = stg_free;  // released once the store has read it (above)
                } else {
                    mbar_arrive(stg_free);
                }
            }
        }
        if (storer && store_free != nullptr) {
            bulk_wait_read_all();
            mbar_arrive(store_free);
        }
        if (storer && stores_issued) bulk_wait_all();  // every tensor store completes before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int KN>
cudaError_t launch_kn(const void *q, const void *k, const void *v, void *out, const BandParams &p,
                      const AttnShape &s, cudaStream_t st)
{
    using Cfg = BandCfg<KN>;
    alignas(64) CUtensorMap mq, mk, mv, mo;
    // fixed-length batches: [B][L][H][D]; packed sequences: [1][total][H][D]
    const uint64_t qrows = s.cu_q ? (uint64_t)s.total_q : (uint64_t)s.Lq;
    const uint64_t krows = s.cu_q ? (uint64_t)s.total_k : (uint64_t)s.Lk;
    const uint64_t outer = s.cu_q ? 1u : (uint64_t)s.B;
    {
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.Hq, qrows, outer};
        const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)s.Hq * kD * 2, qrows * s.Hq * kD * 2};
        const uint32_t box[4] = {(uint32_t)kD, (uint32_t)p.Gp, (uint32_t)p.P, 1u};
        if (!encode_tensor_map_4d(&mq, const_cast<void *>(q), 2, dims, strides, box, true) ||
            !encode_tensor_map_4d(&mo, out, 2, dims, strides, box, true))
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.Hkv, krows, outer};
        const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)s.Hkv * kD * 2, krows * s.Hkv * kD * 2};
        const uint32_t box[4] = {(uint32_t)kD, 1u, (uint32_t)KN, 1u};
        if (!encode_tensor_map_4d(&mk, const_cast<void *>(k), 2, dims, strides, box, true) ||
            !encode_tensor_map_4d(&mv, const_cast<void *>(v), 2, dims, strides, box, true))
            return cudaErrorInvalidValue;
    }
    auto kern = fwd_band_kernel<KN>;
    // The register moves inside the kernel are sized for a launch at exactly
    // kRegsLaunch registers per thread; a build that compiled to fewer would
    // leave the softmax warpgroups waiting for registers that never come.
    static int regs = -1;
    if (regs < 0) {
        cudaFuncAttributes a;
        cudaError_t e = cudaFuncGetAttributes(&a, kern);
        if (e != cudaSuccess) return e;
        regs = a.numRegs;
    }
    if (regs != kRegsLaunch) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<p.n_items, kThreads, Cfg::kSmemBytes, st>>>(mq, mk, mv, mo, p);
    return cudaGetLastError();
}

// query heads packed per item (a power of two dividing the group, at most 16)
int packed_heads(const AttnShape &s)
{
    const int G = s.Hq / s.Hkv;
    int gp = 1;
    while (gp * 2 <= 16 && G % (gp * 2) == 0) gp *= 2;
    return gp;
}

// Keys per tile the shape needs: the band plus the item's positions, rounded up
// to a built tile width (0 when none is wide enough).
int band_tile_keys(const AttnShape &s)
{
    if (s.window <= 0) return 0;
    const long need = (long)s.window + kM / packed_heads(s) - 1;
    const int widths[] = {32, 64, 96, 144};
    for (int w : widths)
        if (need <= w) return w;
    return 0;
}

}  // namespace

bool fwd_band_supported(const AttnShape &s)
{
    return s.D == kD && s.Hq % s.Hkv == 0 && s.window > 0 && band_tile_keys(s) > 0 && s.scale > 0.f;
}

cudaError_t launch_fwd_band(const void *q, const void *k, const void *v, const float *sinks, void *out, float *lse,
                            const AttnShape &s, cudaStream_t st)
{
    BandParams p;
    p.B = s.B;
    p.Lq = s.Lq;
    p.Lk = s.Lk;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.window = s.window;
    p.cu_q = s.cu_q;
    p.cu_k = s.cu_k;
    p.total_q = s.total_q;
    p.total_k = s.total_k;
    p.lse_hs = s.lse_hs > 0 ? s.lse_hs : (s.cu_q ? s.total_q : s.Lq);
    p.G = s.Hq / s.Hkv;
    p.Gp = packed_heads(s);
    p.P = kM / p.Gp;
    p.n_ptiles = (s.Lq + p.P - 1) / p.P;
    p.n_htiles = s.Hq / p.Gp;
    const long long n_items = (long long)p.n_ptiles * p.n_htiles * s.B;
    if (n_items > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.n_items = (int)n_items;
    // the mask's -2^100 times scale * log2(e) must stay far below any exponent
    p.mask_mma = p.P <= 16 && s.scale >= 0x1p-60f;
    p.c_log2 = s.scale * kLog2e;
    p.sinks = sinks;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = device_status_ptr();
    p.timeout_ns = wait_timeout_ns();
    switch (band_tile_keys(s)) {
    case 32: return launch_kn<32>(q, k, v, out, p, s, st);
    case 64: return launch_kn<64>(q, k, v, out, p, s, st);
    case 96: return launch_kn<96>(q, k, v, out, p, s, st);
    case 144: return launch_kn<144>(q, k, v, out, p, s, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn_sink
