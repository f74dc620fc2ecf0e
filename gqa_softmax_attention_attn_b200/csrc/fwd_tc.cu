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
//  * Work item = 128 query rows = (128 / Gp) positions x Gp query heads of one
//    KV group, so every K/V tile fetched is shared by Gp heads (GQA packing;
//    no cluster multicast).  The grid has one CTA per work item, numbered
//    longest first; a running CTA (two per SM, 256 TMEM columns each) takes
//    over the items of CTAs that have not started yet through cluster launch
//    control (the hardware cancels their launch), so a CTA on a faster SM
//    takes more items, and no counter or other state outlives the launch.
//  * Warp 0: item fetch (passed to the other warps through a shared-memory
//    ring) and TMA producer -- Q (double-buffered, so the next item's Q lands
//    while the current one finishes) and K/V tiles of BN keys into an
//    NS-stage ring.  Warp 1: allocates tensor memory and runs the MMA issue
//    loop as a whole warp (warp-uniform descriptors), one elected lane
//    issuing tcgen05.mma: S = Q K^T into a double-buffered TMEM tile, O += P V
//    with P read back from TMEM.  Warps 2-5: one thread per row --
//    tcgen05.ld of S, masking, the exp2 softmax, P written over S as bf16,
//    conditional rescale of O, epilogue.  (Compile-time option SPLIT = 2:
//    warps 2-9, two per row on half the columns each, each half with its own
//    online softmax and O accumulator, combined once per item.)
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

#include <algorithm>
#include <type_traits>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

constexpr int kM = 128;
constexpr int kD = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Banded-layer tile configuration (compile-time knob for measurements)
// (measured on the window-128 layer of the gpt-oss-20b prefill: BN 32 with
// three CTAs per SM 47 us, BN 64 with two 54 us, BN 32 with two 49 us)
#ifndef ATTN_SINK_FWD_BAND_BN
#define ATTN_SINK_FWD_BAND_BN 32
#define ATTN_SINK_FWD_BAND_NS 4
#define ATTN_SINK_FWD_BAND_CPS 3
#endif

// Tile configurations (keys per tile BN, K/V stages NS, EMU = which pair of
// every 4 uses the FMA-pipe exp2 (4: every odd pair, -1: none), CTAs per
// SM), chosen per layer type from measurements on the gpt-oss-20b prefill:
// the dense causal layer runs best with BN = 80, two CTAs per SM and a
// quarter of the exponentials off the MUFU unit (none: 2% slower, half: 7%
// slower), the window-128 layer with the banded configuration above.
// dense layer: BN = 80 with three stages (two CTAs per SM) measured 203 us on
// the gpt-oss-20b prefill's dense layer, against 209 us at BN = 96 and 233 us
// at BN = 64 (and 255-270 us for BN = 32 at three or four CTAs per SM)
#ifndef ATTN_SINK_FWD_DENSE_BN
#define ATTN_SINK_FWD_DENSE_BN 80
#define ATTN_SINK_FWD_DENSE_NS 3
#endif
#ifndef ATTN_SINK_FWD_DENSE_CPS
#define ATTN_SINK_FWD_DENSE_CPS 2
#endif
#ifndef ATTN_SINK_FWD_DENSE_EMU
#define ATTN_SINK_FWD_DENSE_EMU 3
#endif
// softmax warps per row (1 or 2) per layer type; two warps per row (half the
// columns each, each half its own online softmax and O, combined per item)
// measured slower on the gpt-oss-20b prefill's dense layer (234 us at 64-key
// tiles against 207 us), as did trading partial maxima every tile (239 vs 212)
#ifndef ATTN_SINK_FWD_DENSE_SPLIT
#define ATTN_SINK_FWD_DENSE_SPLIT 1
#endif
#ifndef ATTN_SINK_FWD_BAND_SPLIT
#define ATTN_SINK_FWD_BAND_SPLIT 1
#endif
// 1: exponentials against the current reference maximum with the tile maximum
// taken in the same pass (a rare second pass when it moves); 0: the tile
// maximum first, then the exponentials
#ifndef ATTN_SINK_FWD_SPEC
#define ATTN_SINK_FWD_SPEC 1
#endif
constexpr bool FWD_SPEC = ATTN_SINK_FWD_SPEC != 0;
// 1: with FWD_SPEC, the pass tracks no maximum; a tile whose exponentials sum
// past kSumLimit (so one of them may exceed it) takes the rare path, which
// finds the maximum (measured on the gpt-oss-20b prefill's dense layer:
// 208.9 -> 206.9 us); 0: the maximum tracked in the pass, the rare path when
// it exceeds the reference by 2^8
#ifndef ATTN_SINK_FWD_SUMCHECK
#define ATTN_SINK_FWD_SUMCHECK 1
#endif
constexpr bool FWD_SUMCHECK = ATTN_SINK_FWD_SUMCHECK != 0;
constexpr float kSumLimit = 1024.f;
// launch-control requests in flight: dense items are long, so one hides the
// round trip (measured on the gpt-oss-20b prefill's dense layer: 205.6 us at
// one, 206.8 at two, 230.5 at four, where CTAs hold on to items others could
// have taken)
constexpr int kClcDepthDense = 1;
constexpr int pow2_at_least(int x) { return x <= 32 ? 32 : x <= 64 ? 64 : x <= 128 ? 128 : x <= 256 ? 256 : 512; }

// F8: q and k as e4m3 codes (one fp32 scale per query head for q, per KV head
// for k), S = Q K^T on the 8-bit tensor-core path (the products of e4m3
// values are exact, accumulated in fp32); v arrives widened exactly to f16
// (by widen_e4m3_kernel; its scale per KV head multiplies O), so P (f16) V
// runs on the 16-bit path.
template <int BN, int NS, int CPS, int SPLIT, bool F8 = false>
struct FwdCfg {
    static_assert(SPLIT == 1 || SPLIT == 2, "one or two softmax warps per row");
    static_assert(BN % (16 * SPLIT) == 0, "each softmax warp takes whole 16-column chunks");
    static constexpr int kThreads = 64 + 128 * SPLIT;
    static constexpr int kCols = BN / SPLIT;  // score columns per softmax thread
    static constexpr int kEB = F8 ? 1 : 2;  // bytes per q, k element (v is 16-bit either way)
    static constexpr int kQBytes = kM * kD * kEB;
    static constexpr int kKBytes = BN * kD * kEB;
    static constexpr int kVBytes = BN * kD * 2;
    static constexpr int kOffQ = 0;  // two Q buffers
    static constexpr int kOffK = 2 * kQBytes;
    static constexpr int kOffV = kOffK + NS * kKBytes;
    static_assert(kQBytes % 1024 == 0 && kKBytes % 1024 == 0 && kVBytes % 1024 == 0, "tiles on 1024-byte boundaries");
    static constexpr int kOffBar = kOffV + NS * kVBytes;
    // q_full[2], q_empty[2], k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
    // s_full[2], p_full[2], o_done, o_free, drain, xchg[4], item_full[4], item_empty[4], clc[kClcDepthDense]
    static constexpr int kNumBar = 4 + 4 * NS + 4 + 3 + 4 + 8 + kClcDepthDense;
    // tmem slot (+0), abort flag (+4), item ring (+16, 4 ints), launch-control responses (+32, 16 bytes each)
    static constexpr int kOffMisc = (kOffBar + kNumBar * 8 + 15) / 16 * 16;
    static_assert(32 + 16 * kClcDepthDense <= 128, "misc area");
    // row partials exchanged by the two softmax warps of a row: [2 slots][2 halves][128 rows]
    static constexpr int kOffXchg = kOffMisc + 128;
    static constexpr int kTmemCols = pow2_at_least(2 * BN + kD * SPLIT);  // S double buffer + one O per column half
    static constexpr int kCtasPerSm = CPS;  // CTAs resident per SM (TMEM, registers, shared memory)
    static_assert(kTmemCols * CPS <= 512, "tensor memory over-subscribed");
    // + slack for 1024-byte alignment; a CTA that takes all 512 TMEM columns
    // also takes enough shared memory that no second CTA lands on its SM
    static constexpr int kSmemUsed = kOffXchg + 2 * 2 * kM * 4 + 1024;
    static constexpr int kSmemBytes = (kCtasPerSm == 1 && kSmemUsed < 116 * 1024) ? 116 * 1024 : kSmemUsed;
    static constexpr int kTmS0 = 0;
    static constexpr int kTmO = 2 * BN;
};

struct FwdTcParams {
    int B, Lq, Lk, Hq, Hkv, window;
    const int *cu_q, *cu_k;  // packed ragged sequences (else nullptr)
    int total_q, total_k;
    long long lse_hs;        // lse stride between heads: Lq, or total_q for packed sequences
    const float *q_scale, *k_scale, *v_scale;  // F8: per query head, per KV head, per KV head
    int G, Gp, P;  // group size, query heads packed per tile, positions per tile
    int n_ptiles, n_htiles, n_items;
    float c_log2;  // scale * log2(e)
    const float *sinks;
    __nv_bfloat16 *out;
    float *lse;
    unsigned *status;
    long long timeout_ns;
};

struct Item {
    int pos0, h0, b, t_lo, n_tiles;
    int Lq, Lk;        // the sequence's query and key counts
    int qrow0, krow0;  // tensor-map row of its position 0 / key 0
    int tb;            // tensor-map outer coordinate (batch; 0 for packed sequences)
    long long orow0;   // output row of its position 0
    long long lrow0;   // lse index of (head 0, position 0)
    bool empty;        // the item lies past the end of a shorter packed sequence
};

// Work item i of the longest-first order: q tiles from the last (most keys
// under a causal mask) to the first, all head tiles and batches of one q tile
// next to each other.
template <int BN>
__device__ __forceinline__ Item item_at(const FwdTcParams &p, int i)
{
    Item it;
    const int per_q = p.n_htiles * p.B;
    const int qt = p.n_ptiles - 1 - i / per_q;
    const int r = i % per_q;
    it.h0 = (r % p.n_htiles) * p.Gp;
    it.b = r / p.n_htiles;
    it.pos0 = qt * p.P;
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
    const long off = (long)it.Lk - it.Lq;
    const int pos_last = min(it.pos0 + p.P - 1, it.Lq - 1);
    const long lo = p.window > 0 ? max(0L, it.pos0 + off - p.window + 1) : 0L;
    const long hi = min((long)it.Lk, pos_last + off + 1);  // exclusive
    it.t_lo = (int)(lo / BN);
    it.n_tiles = (hi > lo && !it.empty) ? (int)((hi - 1) / BN) - it.t_lo + 1 : 0;
    return it;
}

// Drain wait used on the way out (after an abort too): ignores the abort flag
// and allows at least 1 s whatever the caller's wait limit, so a CTA never
// exits with its own TMA loads or MMAs still in flight.
__device__ __forceinline__ bool wait_noabort(uint64_t *bar, uint32_t parity, unsigned *status, long long tmo)
{
    int never = 0;
    return mbar_wait(bar, parity, &never, status, tmo > 1000000000LL ? tmo : 1000000000LL);
}

template <int BN, int NS, int EMU, int CPS, int SPLIT, bool F8 = false>
__global__ void __launch_bounds__(FwdCfg<BN, NS, CPS, SPLIT, F8>::kThreads, CPS)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdTcParams p)
{
    using Cfg = FwdCfg<BN, NS, CPS, SPLIT, F8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *q_full = bars;
    uint64_t *q_empty = bars + 2;
    uint64_t *k_full = bars + 4;
    uint64_t *k_empty = k_full + NS;
    uint64_t *v_full = k_empty + NS;
    uint64_t *v_empty = v_full + NS;
    uint64_t *s_full = v_empty + NS;
    uint64_t *p_full = s_full + 2;
    uint64_t *o_done = p_full + 2;
    uint64_t *o_free = o_done + 1;
    uint64_t *drain = o_free + 1;
    uint64_t *xchg = drain + 1;  // [4]: one per TMEM lane quadrant (SPLIT == 2)
    // item ring (dynamic order): the producer warp fetches items and passes
    // them to the MMA warp and the softmax warps through 4 slots
    uint64_t *item_full = xchg + 4;        // [4]
    uint64_t *item_empty = item_full + 4;  // [4]
    uint64_t *clc_bar = item_empty + 4;    // [kClcDepthDense]: launch-control responses landed
    volatile int *ring = reinterpret_cast<volatile int *>(smem + Cfg::kOffMisc + 16);
    void *clc_resp = smem + Cfg::kOffMisc + 32;
    float *xs = reinterpret_cast<float *>(smem + Cfg::kOffXchg);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Cfg::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 128 * SPLIT);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(o_done, 1);
        mbar_init(o_free, 128 * SPLIT);
        mbar_init(drain, 1);
        for (int qd = 0; qd < 4; ++qd) mbar_init(&xchg[qd], 64);
        for (int r = 0; r < 4; ++r) {
            mbar_init(&item_full[r], 1);
            mbar_init(&item_empty[r], 1 + 4 * SPLIT);  // the MMA warp and each softmax warp
        }
        for (int d = 0; d < kClcDepthDense; ++d) mbar_init(&clc_bar[d], 1);
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

    // r-th item of this CTA: its own (blockIdx.x) first, then the items of the
    // CTAs whose launch it cancels.  The producer (lane 0 of warp 0) learns
    // it, requests the next one at once (so the request's latency hides behind
    // the item) and publishes it in the ring; every other warp reads it there
    // (-1: no more).  Items past the end of a shorter packed sequence are
    // passed over here, so the other warps never see them.
    ClcQueue<kClcDepthDense> clc{clc_bar, reinterpret_cast<uint8_t *>(clc_resp)};
    auto producer_item = [&](int r) -> int {
        int w = r == 0 ? (int)blockIdx.x : clc.next(abort_flag, p.status, p.timeout_ns);
        clc.fill();  // keep kClcDepthDense requests in flight
        while (w >= 0 && item_at<BN>(p, w).empty) {
            w = clc.next(abort_flag, p.status, p.timeout_ns);
            clc.fill();
        }
        if (clc.failed) return -1;
        const int sl = r & 3;
        if (!mbar_wait(&item_empty[sl], ((r >> 2) & 1u) ^ 1u, abort_flag, p.status, p.timeout_ns)) return -1;
        ring[sl] = w;
        mbar_arrive(&item_full[sl]);
        return w;
    };
    auto consumer_item = [&](int r) -> int {
        const int sl = r & 3;
        if (!__all_sync(0xffffffffu, mbar_wait(&item_full[sl], (r >> 2) & 1u, abort_flag, p.status, p.timeout_ns)))
            return -1;
        const int w = ring[sl];
        __syncwarp();
        if (lane == 0) mbar_arrive(&item_empty[sl]);
        return w;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // e4m3 inputs: v comes widened from the kernel ahead, whose grid
            // lets this one start early (programmatic dependent launch); the
            // loads wait for it (no-op for a grid launched the plain way)
            if (F8) grid_dep_wait();
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            uint32_t k_issued[NS], v_issued[NS], q_issued[2] = {0, 0};
            for (int s = 0; s < NS; ++s) k_issued[s] = v_issued[s] = 0;
            uint32_t it = 0, item_n = 0;
            bool ok = true;
            for (int r_it = 0, w = producer_item(0); w >= 0 && ok; w = producer_item(++r_it)) {
                const Item t = item_at<BN>(p, w);
                if (t.n_tiles == 0) continue;
                const int qb = item_n & 1;
                if (!mbar_wait(&q_empty[qb], ((item_n >> 1) & 1u) ^ 1u, abort_flag, p.status, p.timeout_ns)) break;
                mbar_arrive_expect_tx(&q_full[qb], Cfg::kQBytes);
                tma_load_4d(smem + Cfg::kOffQ + qb * Cfg::kQBytes, &tmQ, 0, t.h0, t.qrow0 + t.pos0, t.tb,
                            &q_full[qb]);
                ++q_issued[qb];
                const int g = t.h0 / p.G;
                for (int jt = 0; jt < t.n_tiles; ++jt, ++it) {
                    const int st = it % NS;
                    const uint32_t ph = (it / NS) & 1u;
                    const int j0 = (t.t_lo + jt) * BN;
                    if (!mbar_wait(&k_empty[st], ph ^ 1u, abort_flag, p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&k_full[st], Cfg::kKBytes);
                    tma_load_4d(smem + Cfg::kOffK + st * Cfg::kKBytes, &tmK, 0, g, t.krow0 + j0, t.tb, &k_full[st]);
                    ++k_issued[st];
                    if (!mbar_wait(&v_empty[st], ph ^ 1u, abort_flag, p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&v_full[st], Cfg::kVBytes);
                    tma_load_4d(smem + Cfg::kOffV + st * Cfg::kVBytes, &tmV, 0, g, t.krow0 + j0, t.tb, &v_full[st]);
                    ++v_issued[st];
                }
                ++item_n;
            }
            // every load issued, and a launch-control request still in flight,
            // must land before the CTA may exit
            clc.drain(p.status, p.timeout_ns);
            for (int s = 0; s < 2; ++s)
                if (q_issued[s]) wait_noabort(&q_full[s], (q_issued[s] - 1) & 1u, p.status, p.timeout_ns);
            for (int s = 0; s < NS; ++s) {
                if (k_issued[s]) wait_noabort(&k_full[s], (k_issued[s] - 1) & 1u, p.status, p.timeout_ns);
                if (v_issued[s]) wait_noabort(&v_full[s], (v_issued[s] - 1) & 1u, p.status, p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop (so every operand is warp-uniform) and
        // one elected lane issues the MMAs and their commits.
        const uint32_t id_s = F8 ? idesc_e4m3_f32(kM, BN) : idesc_bf16_f32(kM, BN, 0);
        const uint32_t id_pv = F8 ? idesc_f16_f32(kM, kD, 1) : idesc_bf16_f32(kM, kD, 1);
        const uint32_t k_addr = smem_u32(smem + Cfg::kOffK);
        const uint32_t v_addr = smem_u32(smem + Cfg::kOffV);
        auto wait_all = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status, p.timeout_ns));
        };
        uint32_t it = 0, item_n = 0;
        bool ok = true;
        // O += P(t) V(t); the first product of an item overwrites O, which
        // must wait until the previous item's epilogue has read O out.
        auto issue_pv = [&](uint32_t t, bool first) -> bool {
            const int sb = t & 1, st = t % NS;
            if (first && !wait_all(o_free, (item_n & 1u) ^ 1u)) return false;
            if (!wait_all(&p_full[sb], (t >> 1) & 1u)) return false;
            if (!wait_all(&v_full[st], (t / NS) & 1u)) return false;
            tc_fence_after();
            const uint32_t vb = v_addr + st * Cfg::kVBytes;
            if (elect_one()) {
                // V tile [BN keys][64 d] is the MN-major B operand: 16 keys = 2048 bytes per step.
                // Column half hh's P (its 16-key blocks, bf16 pairs at the start of its own
                // S columns) goes into its own O accumulator.
#pragma unroll
                for (int hh = 0; hh < SPLIT; ++hh)
#pragma unroll
                    for (int kk = 0; kk < BN / 16 / SPLIT; ++kk) {
                        const int kb = hh * (BN / 16 / SPLIT) + kk;  // 16-key block of the tile
                        const uint64_t bdesc = smem_desc_sw128(vb + kb * 2048, BN * 128, 1024);
                        mma_ts(tmem + Cfg::kTmO + kD * hh, tmem + Cfg::kTmS0 + sb * BN + hh * Cfg::kCols + kk * 8,
                               bdesc, id_pv, (!first || kk > 0) ? 1u : 0u);
                    }
                mma_commit(o_done);
                mma_commit(&v_empty[st]);
            }
            __syncwarp();
            return true;
        };
        for (int r_it = 0, w = consumer_item(0); w >= 0 && ok; w = consumer_item(++r_it)) {
            const Item t = item_at<BN>(p, w);
            if (t.n_tiles == 0) continue;
            const int qb = item_n & 1;
            if (!wait_all(&q_full[qb], (item_n >> 1) & 1u)) break;
            tc_fence_after();
            const uint32_t q_addr = smem_u32(smem + Cfg::kOffQ + qb * Cfg::kQBytes);
            for (int jt = 0; jt < t.n_tiles; ++jt, ++it) {
                const int st = it % NS, sb = it & 1;
                if (!wait_all(&k_full[st], (it / NS) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t kb = k_addr + st * Cfg::kKBytes;
                if (elect_one()) {
                    if (F8) {
                        // e4m3 rows of 64 bytes, 64-byte swizzle: K = 32 codes (32 bytes) per step
#pragma unroll
                        for (int kk = 0; kk < kD / 32; ++kk)
                            mma_ss_f8(tmem + Cfg::kTmS0 + sb * BN, smem_desc_sw64(q_addr + kk * 32, 512),
                                      smem_desc_sw64(kb + kk * 32, 512), id_s, kk > 0 ? 1u : 0u);
                    } else {
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(q_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(kb + kk * 32, 16, 1024);
                        mma_ss(tmem + Cfg::kTmS0 + sb * BN, adesc, bdesc, id_s, kk > 0 ? 1u : 0u);
                    }
                    }
                    mma_commit(&s_full[sb]);
                    mma_commit(&k_empty[st]);
                    if (jt == t.n_tiles - 1) mma_commit(&q_empty[qb]);
                }
                __syncwarp();
                if (jt >= 1 && !issue_pv(it - 1, jt == 1)) {
                    ok = false;
                    break;
                }
            }
            if (!ok || !issue_pv(it - 1, t.n_tiles == 1)) {
                ok = false;
                break;
            }
            ++item_n;
        }
        if (elect_one()) mma_commit(drain);
        __syncwarp();
        wait_noabort(drain, 0, p.status, p.timeout_ns);
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        // SPLIT warps per row: the warp of column half h (warps 2-5: h = 0,
        // warps 6-9: h = 1) takes score columns [h kCols, (h + 1) kCols) of
        // each tile and runs its own online softmax over them (its own
        // reference maximum, sum and O accumulator; the sink seeds half 0).
        // At the end of an item the two halves trade their maxima and sums
        // through shared memory, ordered by the quadrant's exchange barrier,
        // combine O0 and O1 and write columns [h 64 / SPLIT, ...) each --
        // exact, since each half's numerator and denominator share its own
        // reference.
        constexpr int kC = Cfg::kCols;
        constexpr int kOC = kD / SPLIT;  // O columns per thread
        const int quad = warp & 3;
        const int half = SPLIT == 2 ? (warp - 2) >> 2 : 0;
        const int r = quad * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        float C = p.c_log2;  // F8: times the row's q and k scales (set per item)
        uint32_t it = 0, xc = 0;
        bool ok = true;
        // publish v, get the other half's value (bounded wait; false on abort)
        auto trade = [&](float v, float &other) -> bool {
            const int slot = xc & 1;
            xs[(slot * 2 + half) * kM + r] = v;
            mbar_arrive(&xchg[quad]);
            const bool got =
                __all_sync(0xffffffffu, mbar_wait(&xchg[quad], xc & 1u, abort_flag, p.status, p.timeout_ns));
            other = xs[(slot * 2 + (half ^ 1)) * kM + r];
            ++xc;
            return got;
        };
        for (int r_it = 0, w = consumer_item(0); w >= 0 && ok; w = consumer_item(++r_it)) {
            const Item t = item_at<BN>(p, w);
            const int pos = t.pos0 + r / p.Gp;
            const int h = t.h0 + r % p.Gp;
            const bool row_valid = pos < t.Lq;
            const long pabs = pos + ((long)t.Lk - t.Lq);
            const float sink2 = p.sinks[h] * kLog2e;  // the sink logit in log2 units
            if (F8) C = p.c_log2 * p.q_scale[h] * p.k_scale[h / p.G];
            float m = half == 0 ? sink2 : -INFINITY;   // reference maximum, log2 units
            // running sum, seeded with the sink's mass (in column half 0 only)
            float l = (sink2 == -INFINITY || half != 0) ? 0.f : 1.f;
            // rows beyond Lq only need finite, unused values
            const long vis_hi = row_valid ? min(pabs, (long)t.Lk - 1) : -1;   // last visible key
            const long vis_lo = p.window > 0 ? pabs - p.window + 1 : 0;     // first visible key

            for (int jt = 0; jt < t.n_tiles; ++jt, ++it) {
                const int sb = it & 1;
                const long j0 = (long)(t.t_lo + jt) * BN + half * kC;  // first key of this thread's columns
                if (!__all_sync(0xffffffffu,
                                mbar_wait(&s_full[sb], (it >> 1) & 1u, abort_flag, p.status, p.timeout_ns))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t scol = Cfg::kTmS0 + sb * BN + half * kC;
                uint32_t sr[kC / 16][16];
#pragma unroll
                for (int c = 0; c < kC / 16; ++c) tmem_ld16(trow + scol + c * 16, sr[c]);
                tmem_wait_ld();
                float sv[kC];
#pragma unroll
                for (int c = 0; c < kC; ++c) sv[c] = __uint_as_float(sr[c / 16][c % 16]);
                // visible columns of this thread: c in [c_lo, c_hi] (32-bit, relative to j0)
                const int c_hi = (int)max(-1L, min((long)kC - 1, vis_hi - j0));
                const int c_lo = (int)max(0L, min((long)kC, vis_lo - j0));
                const bool need_mask = __any_sync(0xffffffffu, c_lo > 0 || c_hi < kC - 1);
                if (need_mask) {
#pragma unroll
                    for (int c = 0; c < kC; ++c) sv[c] = (c >= c_lo && c <= c_hi) ? sv[c] : -INFINITY;
                }
                static_assert(kC % 16 == 0, "whole 16-column chunks per thread");
                const float2 C2 = make_float2(C, C);
                float2 acc[2];
                float mx[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
                // One pass over the tile: P = exp2(S C - m) against the reference
                // maximum m, written as bf16 pairs over the first kC/2 columns of
                // this thread's part of the S buffer (read in full already), 16
                // scores per store; with kTrack, the tile's row maximum too, in
                // eight independent chains of 3-input max.  On tiles with no
                // masked element, pair EMU of every 4 runs on the FMA pipe
                // (fast_exp2x2) to offload the MUFU unit.
                auto exp_pass = [&](float neg_m_, auto track_tag, auto emu_tag) {
                    constexpr bool kTrack = decltype(track_tag)::value;
                    constexpr bool kEmu = decltype(emu_tag)::value;
                    const float2 M2 = make_float2(neg_m_, neg_m_);
                    acc[0] = acc[1] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < kC / 16; ++c) {
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float2 x = ffma2(make_float2(sv[16 * c + 2 * e], sv[16 * c + 2 * e + 1]), C2, M2);
                            const bool emu = kEmu && (EMU == 4 ? (e & 1) != 0 : (e & 3) == EMU);
                            const float2 pe = emu ? fast_exp2x2(x) : make_float2(ex2(x.x), ex2(x.y));
                            acc[e & 1] = fadd2(acc[e & 1], pe);
                            pk[e] = F8 ? pack_f16x2(pe.x, pe.y) : pack_bf16x2(pe.x, pe.y);
                        }
                        if (kTrack) {
#pragma unroll
                            for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], sv[16 * c + k], sv[16 * c + 8 + k]);
                        }
                        tmem_st8(trow + scol + c * 8, pk);
                    }
                };
                bool rescale = false;
                float alpha = 1.f;
                if (FWD_SPEC) {
                    // The exponentials first, against the current reference (it
                    // only moves when a tile's exponentials grow past a bound, so
                    // it rarely does); a row whose reference does move redoes the
                    // pass (S is still in registers, P not yet handed to the MMA).
                    const float neg_m0 = (m == -INFINITY) ? 0.f : -m;
                    float m_new = m;
                    if (FWD_SUMCHECK) {
                        if (need_mask)
                            exp_pass(neg_m0, std::false_type{}, std::false_type{});
                        else
                            exp_pass(neg_m0, std::false_type{}, std::true_type{});
                        // every exponential is at most their sum: a sum within
                        // kSumLimit (NaN fails the test) keeps the reference; a
                        // row with no reference yet (sink -inf) takes the rare
                        // path until a tile gives it one
                        const float tsum = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
                        const bool big = !(tsum <= kSumLimit) || m == -INFINITY;
                        if (__any_sync(0xffffffffu, big)) {
#pragma unroll
                            for (int c = 0; c < kC; c += 16)
#pragma unroll
                                for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], sv[c + k], sv[c + 8 + k]);
                            const float tmax =
                                fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
                            m_new = fmaxf(m, tmax * C);
                            rescale = big && m_new > m;
                        }
                    } else {
                        if (need_mask)
                            exp_pass(neg_m0, std::true_type{}, std::false_type{});
                        else
                            exp_pass(neg_m0, std::true_type{}, std::true_type{});
                        const float tmax =
                            fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
                        m_new = fmaxf(m, tmax * C);
                        rescale = m_new > m + kRescaleThreshold;
                    }
                    if (__any_sync(0xffffffffu, rescale)) {
                        alpha = rescale ? ((m == -INFINITY) ? 0.f : ex2(m - m_new)) : 1.f;
                        if (rescale) m = m_new;
                        exp_pass((m == -INFINITY) ? 0.f : -m, std::false_type{}, std::false_type{});
                    }
                } else {
                    // the tile's row maximum first, then the exponentials
#pragma unroll
                    for (int c = 0; c < kC; c += 16)
#pragma unroll
                        for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], sv[c + k], sv[c + 8 + k]);
                    float tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
                    const float m_new = fmaxf(m, tmax * C);
                    rescale = m_new > m + kRescaleThreshold;
                    alpha = rescale ? ((m == -INFINITY) ? 0.f : ex2(m - m_new)) : 1.f;
                    if (rescale) m = m_new;
                    const float neg_m = (m == -INFINITY) ? 0.f : -m;
                    if (need_mask)
                        exp_pass(neg_m, std::false_type{}, std::false_type{});
                    else
                        exp_pass(neg_m, std::false_type{}, std::true_type{});
                }
                l = l * alpha + ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y));
                if (jt > 0) {
                    // O holds sum_{t<jt} P_t V_t once PV(jt-1) completes.  Waited on
                    // every tile, rescale or not: a parity wait is only unambiguous
                    // while the barrier is at most one phase away, so no phase of
                    // o_done may go unobserved.
                    if (!__all_sync(0xffffffffu,
                                    mbar_wait(o_done, (it - 1) & 1u, abort_flag, p.status, p.timeout_ns))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, rescale)) {
                        // this half's own O accumulator (all 64 columns)
                        uint32_t o[kD / 32][32];
#pragma unroll
                        for (int c = 0; c < kD / 32; ++c) tmem_ld32(trow + Cfg::kTmO + kD * half + 32 * c, o[c]);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < kD; ++c)
                            o[c / 32][c % 32] = __float_as_uint(__uint_as_float(o[c / 32][c % 32]) * alpha);
#pragma unroll
                        for (int c = 0; c < kD / 32; ++c) tmem_st32(trow + Cfg::kTmO + kD * half + 32 * c, o[c]);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[sb]);
            }
            if (!ok) break;

            // -------------------------------------------------------- epilogue
            uint32_t o[kOC / 32][32];
            float a_me = 1.f, a_ot = 0.f;  // SPLIT == 2: weights of this half's and the other half's O
            if (SPLIT == 2) {
                // the two halves' reference maxima and sums -> one reference M
                float m_o, l_o;
                if (!trade(m, m_o) || !trade(l, l_o)) {
                    ok = false;
                    break;
                }
                const float M = fmaxf(m, m_o);
                a_me = (m == -INFINITY) ? 0.f : ex2(m - M);
                a_ot = (m_o == -INFINITY) ? 0.f : ex2(m_o - M);
                l = l * a_me + l_o * a_ot;
                m = M;
            }
            if (t.n_tiles > 0) {
                if (!__all_sync(0xffffffffu,
                                mbar_wait(o_done, (it - 1) & 1u, abort_flag, p.status, p.timeout_ns))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (SPLIT == 2) {
                    // columns [32 half, 32 half + 32) of both halves' O
                    uint32_t o0[32], o1[32];
                    tmem_ld32(trow + Cfg::kTmO + 32 * half, o0);
                    tmem_ld32(trow + Cfg::kTmO + kD + 32 * half, o1);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(o_free);  // the next item's first PV may overwrite O now
                    const float a0 = half == 0 ? a_me : a_ot, a1 = half == 0 ? a_ot : a_me;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        o[0][c] = __float_as_uint(__uint_as_float(o0[c]) * a0 + __uint_as_float(o1[c]) * a1);
                } else {
#pragma unroll
                    for (int c = 0; c < kOC / 32; ++c) tmem_ld32(trow + Cfg::kTmO + 32 * c, o[c]);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(o_free);  // the next item's first PV may overwrite O now
                }
            } else {
#pragma unroll
                for (int c = 0; c < kOC; ++c) o[c / 32][c % 32] = 0u;
            }
            if (row_valid) {
                const float inv = l > 0.f ? (F8 ? p.v_scale[h / p.G] : 1.f) / l : 0.f;
                uint4 *dst =
                    reinterpret_cast<uint4 *>(p.out + ((size_t)(t.orow0 + pos) * p.Hq + h) * kD + half * kOC);
#pragma unroll
                for (int c = 0; c < kOC / 8; ++c) {
                    const uint32_t *src = &o[c / 4][(c % 4) * 8];
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(src[0]) * inv, __uint_as_float(src[1]) * inv);
                    v.y = pack_bf16x2(__uint_as_float(src[2]) * inv, __uint_as_float(src[3]) * inv);
                    v.z = pack_bf16x2(__uint_as_float(src[4]) * inv, __uint_as_float(src[5]) * inv);
                    v.w = pack_bf16x2(__uint_as_float(src[6]) * inv, __uint_as_float(src[7]) * inv);
                    dst[c] = v;
                }
                if (half == 0)
                    p.lse[(size_t)(t.lrow0 + (long long)h * p.lse_hs + pos)] =
                        l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
            }
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

template <int BN, int NS, int EMU, int CPS, int SPLIT, bool F8 = false>
cudaError_t launch_cfg(const void *q, const void *k, const void *v, const float *sinks, void *out, float *lse,
                       const AttnShape &s, cudaStream_t st, const float *q_scale = nullptr,
                       const float *k_scale = nullptr, const float *v_scale = nullptr)
{
    using Cfg = FwdCfg<BN, NS, CPS, SPLIT, F8>;
    FwdTcParams p;
    p.q_scale = q_scale;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
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
    int gp = 1;
    while (gp * 2 <= 16 && p.G % (gp * 2) == 0) gp *= 2;
    p.Gp = gp;
    p.P = kM / gp;
    p.n_ptiles = (s.Lq + p.P - 1) / p.P;
    p.n_htiles = s.Hq / gp;
    const long long n_items = (long long)p.n_ptiles * p.n_htiles * s.B;
    if (n_items > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.n_items = (int)n_items;
    p.c_log2 = s.scale * kLog2e;
    p.sinks = sinks;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = device_status_ptr();
    p.timeout_ns = wait_timeout_ns();

    alignas(64) CUtensorMap mq, mk, mv;
    // fixed-length batches: [B][L][H][D]; packed sequences: [1][total][H][D]
    const uint64_t qrows = s.cu_q ? (uint64_t)s.total_q : (uint64_t)s.Lq;
    const uint64_t krows = s.cu_q ? (uint64_t)s.total_k : (uint64_t)s.Lk;
    const uint64_t outer = s.cu_q ? 1u : (uint64_t)s.B;
    // bf16: 128-byte rows, 128-byte swizzle; e4m3 q and k: 64-byte rows,
    // 64-byte swizzle; v (bf16, or f16 widened from e4m3) as bf16
    constexpr int eb = Cfg::kEB;
    constexpr int swz_qk = F8 ? 64 : 128;
    {
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.Hq, qrows, outer};
        const uint64_t strides[3] = {(uint64_t)kD * eb, (uint64_t)s.Hq * kD * eb, qrows * s.Hq * kD * eb};
        const uint32_t box[4] = {(uint32_t)kD, (uint32_t)p.Gp, (uint32_t)p.P, 1u};
        if (!encode_tensor_map_4d_sw(&mq, const_cast<void *>(q), eb, dims, strides, box, swz_qk))
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.Hkv, krows, outer};
        const uint64_t strides[3] = {(uint64_t)kD * eb, (uint64_t)s.Hkv * kD * eb, krows * s.Hkv * kD * eb};
        const uint32_t box[4] = {(uint32_t)kD, 1u, (uint32_t)BN, 1u};
        if (!encode_tensor_map_4d_sw(&mk, const_cast<void *>(k), eb, dims, strides, box, swz_qk))
            return cudaErrorInvalidValue;
        const uint64_t vstrides[3] = {(uint64_t)kD * 2, (uint64_t)s.Hkv * kD * 2, krows * s.Hkv * kD * 2};
        if (!encode_tensor_map_4d_sw(&mv, const_cast<void *>(v), 2, dims, vstrides, box, 128))
            return cudaErrorInvalidValue;
    }
    auto kern = fwd_tc_kernel<BN, NS, EMU, CPS, SPLIT, F8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    // one CTA per item: as many start as fit (kCtasPerSm per SM), the rest are
    // taken over by running CTAs before they launch
    if (!F8) {
        kern<<<p.n_items, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mq, mk, mv, p);
        return cudaGetLastError();
    }
    // e4m3: chained to the widening kernel (programmatic dependent launch)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.n_items);
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, p);
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
    if (fwd_band_supported(s)) return launch_fwd_band(q, k, v, sinks, out, lse, s, st);
    if (s.window > 0 && s.window <= 1024)
        return launch_cfg<ATTN_SINK_FWD_BAND_BN, ATTN_SINK_FWD_BAND_NS, -1, ATTN_SINK_FWD_BAND_CPS,
                          ATTN_SINK_FWD_BAND_SPLIT>(q, k, v, sinks, out, lse, s, st);
    return launch_cfg<ATTN_SINK_FWD_DENSE_BN, ATTN_SINK_FWD_DENSE_NS, ATTN_SINK_FWD_DENSE_EMU, ATTN_SINK_FWD_DENSE_CPS,
                      ATTN_SINK_FWD_DENSE_SPLIT>(q, k, v, sinks, out, lse, s, st);
}

namespace {
// e4m3 -> f16, exactly (16 codes per thread, 16-byte loads, 32-byte stores)
__global__ void __launch_bounds__(256) widen_e4m3_kernel(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                                                         size_t n16)
{
    grid_dep_launch();  // the attention kernel may start its set-up
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n16) return;
    uint4 lo, hi;
    e4m3x16_to_f16(reinterpret_cast<const uint4 *>(src)[i], lo, hi);
    reinterpret_cast<uint4 *>(dst)[2 * i] = lo;
    reinterpret_cast<uint4 *>(dst)[2 * i + 1] = hi;
}
}  // namespace

size_t fwd_fp8_workspace_bytes(const AttnShape &s) { return (size_t)s.B * s.Lk * s.Hkv * s.D * 2; }

cudaError_t launch_fwd_tc_fp8(const void *q, const void *k, const void *v, const float *q_scale,
                              const float *k_scale, const float *v_scale, const float *sinks, void *out, float *lse,
                              void *v16, const AttnShape &s, cudaStream_t st)
{
    if (s.cu_q) return cudaErrorInvalidValue;  // fixed-length batches only
    // v widened once into the workspace; the attention kernels read it as 16-bit tiles
    const size_t n16 = (size_t)s.B * s.Lk * s.Hkv * s.D / 16;
    if ((n16 + 255) / 256 > 0x7fffffffu) return cudaErrorInvalidValue;
    if (n16 > 0) {
        widen_e4m3_kernel<<<(unsigned)((n16 + 255) / 256), 256, 0, st>>>(static_cast<const uint8_t *>(v),
                                                                        static_cast<uint8_t *>(v16), n16);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (s.window > 0 && s.window <= 1024)
        return launch_cfg<ATTN_SINK_FWD_BAND_BN, ATTN_SINK_FWD_BAND_NS, -1, ATTN_SINK_FWD_BAND_CPS, 1, true>(
            q, k, v16, sinks, out, lse, s, st, q_scale, k_scale, v_scale);
    return launch_cfg<ATTN_SINK_FWD_DENSE_BN, ATTN_SINK_FWD_DENSE_NS, ATTN_SINK_FWD_DENSE_EMU, ATTN_SINK_FWD_DENSE_CPS,
                      1, true>(q, k, v16, sinks, out, lse, s, st, q_scale, k_scale, v_scale);
}

}  // namespace attn_sink
