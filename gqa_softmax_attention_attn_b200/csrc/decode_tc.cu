// decode_tc.cu -- bf16 split-KV decode of sink-softmax GQA attention.
//
// What it computes ("GPT-OSS on day 0", section "Sink Attention"): one query
// per sequence against that sequence's cached keys, with the work split both
// across KV heads and along the KV length; each split produces a partial
// (running max m, running sum l, unnormalised output o) WITHOUT the sink, and
// the sink joins exactly once, when the splits are combined (or directly here
// when a sequence needs only one split).
//
// Design (B200): the path is HBM-bound (8 flop per byte of KV at GQA group 8).
//  * CTA = (split c, KV head g, sequence b).  Warp 0 streams the split's K and
//    V rows of head g with 2-D-tiled TMA boxes (64 keys x 128 bytes, 128-byte
//    swizzle) into a shared-memory ring (4 stages; 3 for short splits and for
//    paged caches, so four CTAs share an SM); every byte of KV is read from
//    HBM once, for all G query heads of the group.
//  * Warps 1-4 take 16 keys of each 64-key tile: the G query heads of the
//    group (padded to 16 rows) are scored with mma.sync m16n8k16 -- FP32 CUDA
//    cores cannot sustain 8 flop/byte at HBM rate -- then an exp2 online
//    softmax in registers and P V with mma.sync again (P reused from the
//    score accumulators).
//  * Keys past the chunk (ragged tail, cache rows beyond the sequence, or
//    TMA zero fill past Lmax) are masked, and their V rows are zeroed in the
//    operand registers so stale cache contents can never reach the output.
//  * Paged caches (kPaged): K/V live in a pool of pages [num_pages,
//    page_size, Hkv, D] addressed through a per-sequence page table.  Tiles
//    then start on multiples of 64 keys (the split range begins at the
//    visible start rounded down, the keys below it masked), so a tile lies in
//    one page (page_size a multiple of 64) or is 64 / page_size whole pages
//    (page_size 8, 16 or 32), each fetched with its own TMA box.
//  * Every wait is bounded; on expiry the CTA raises the device status bit
//    and winds down.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>

#include <type_traits>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace attn_sink {
namespace {

constexpr int kD = 64;
// K/V ring stages: the loads in flight per SM must cover the HBM latency at
// full bandwidth, so the e4m3 ring (half the bytes per stage) is deeper
#ifndef ATTN_SINK_DEC_FP8_STAGES
#define ATTN_SINK_DEC_FP8_STAGES 3
#endif
constexpr int kThreads = 160;  // warp 0 producer, warps 1-4 consumers
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Shared-memory layout; kFp8: K/V cached as e4m3 (one byte per element).
// kStages: TMA ring depth (bf16: 4, or 3 when a split spans at most three
// tiles, so that more CTAs fit an SM at once; e4m3: ATTN_SINK_DEC_FP8_STAGES)
template <bool kFp8, int kStages>
struct DecLayout {
    // keys per tile: the e4m3 tile spans twice the keys, so a tile's bytes (and
    // its fixed costs: TMA issue, barrier round trips) are those of a bf16 tile
    static constexpr int kT = kFp8 ? 128 : 64;
    static constexpr int kSlices = kT / 64;  // 16-key slices per consumer warp and tile
    static constexpr int kNS = kStages;
    static constexpr int kRowBytes = kFp8 ? kD : kD * 2;  // one cached K or V row
    static constexpr int kTileBytes = kT * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;  // K and V
    // e4m3 only: each consumer warp's keys of V as f16, 128-byte swizzled
    // (K is read straight from the e4m3 tile)
    static constexpr int kOffStaging = kNS * kStageBytes;
    static constexpr int kWarpStaging = kSlices * 16 * kD * 2;
    static constexpr int kOffBar = kOffStaging + (kFp8 ? 4 * kWarpStaging : 0);
    static constexpr int kSmemBytes = kOffBar + 2 * kNS * 8 + 16 + 1024;
    // the final reduction reuses [0, kOffBar): 4 warps x 16 rows x 66 floats
    static_assert(4 * 16 * 66 * 4 <= kOffBar, "reduction buffer");
};

struct DecodeParams {
    DecodeShape sh;  // split rule and (for kPaged) the page pool
    int box_rows;    // rows per TMA box: 64, or page_size when the pages are smaller
    int B, Lmax, Hq, Hkv, G, window, splits, chunk;
    float c_log2;
    const float *k_scale, *v_scale;  // e4m3 caches: per-KV-head dequantisation scales
    const __nv_bfloat16 *q;
    const int *seqlens;
    const float *sinks;
    __nv_bfloat16 *out;
    float *lse;
    float *ws_o, *ws_ml;
    unsigned *status;
    long long timeout_ns;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D (fp32 16x8) += A (bf16 16x16, row) * B (bf16 16x8, col)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D (fp32 16x8) += A (f16 16x16, row) * B (f16 16x8, col)
__device__ __forceinline__ void mma16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of (row, 16-byte chunk) in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }


template <bool kRows16, bool kPaged, bool kFp8, int kStages>
__device__ __forceinline__ void decode_tc_body(const CUtensorMap &tmK, const CUtensorMap &tmV, const DecodeParams &p)
{
    grid_dep_launch();  // the split combine may be launched now; it waits for this grid
    using L = DecLayout<kFp8, kStages>;
    constexpr int kT = L::kT;
    static_assert(!(kPaged && kFp8), "paged caches are bf16 only");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int kNS = L::kNS;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *empty = full + kNS;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffBar + 2 * kNS * 8);

    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int len = min(max(p.seqlens[b], 1), p.Lmax);
    int lo, lo_al, nsplit;
    decode_range(p.sh, len, lo, lo_al, nsplit);
    if (c >= nsplit) return;  // uniform over the CTA
    const int kbeg = lo_al + c * p.chunk;
    const int kend = min(len, kbeg + p.chunk);
    const int n_tiles = (kend - kbeg + kT - 1) / kT;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // per-warp partial state, combined through shared memory at the end
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            uint32_t issued[kNS];
#pragma unroll
            for (int s = 0; s < kNS; ++s) issued[s] = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int st = j % kNS;
                if (!mbar_wait(&empty[st], ((j / kNS) & 1u) ^ 1u, abort_flag, p.status, p.timeout_ns)) break;
                mbar_arrive_expect_tx(&full[st], L::kStageBytes);
                if (kPaged) {
                    // the tile's keys in boxes of box_rows rows, each inside one page;
                    // pages past the sequence (masked keys) reuse its last page, so the
                    // page table is only read within this sequence's own entries
                    const int ps = p.sh.page_size;
                    const int npg = (len + ps - 1) / ps;
                    for (int r0 = 0; r0 < kT; r0 += p.box_rows) {
                        const int key = kbeg + j * kT + r0;
                        const int lp = min(key / ps, npg - 1);
                        const int phys = p.sh.page_table[(size_t)b * p.sh.max_pages + lp];
                        const int slot = key % ps;
                        tma_load_4d(smem + st * L::kStageBytes + r0 * L::kRowBytes, &tmK, 0, g, slot, phys,
                                    &full[st]);
                        tma_load_4d(smem + st * L::kStageBytes + L::kTileBytes + r0 * L::kRowBytes, &tmV, 0, g,
                                    slot, phys, &full[st]);
                    }
                } else {
                    tma_load_4d(smem + st * L::kStageBytes, &tmK, 0, g, kbeg + j * kT, b, &full[st]);
                    tma_load_4d(smem + st * L::kStageBytes + L::kTileBytes, &tmV, 0, g, kbeg + j * kT, b,
                                &full[st]);
                }
                ++issued[st];
            }
            // drain: every issued load lands before the CTA exits (>= 1 s limit, abort ignored)
            for (int s = 0; s < kNS; ++s)
                if (issued[s]) {
                    int never = 0;
                    mbar_wait(&full[s], (issued[s] - 1) & 1u, &never, p.status,
                              p.timeout_ns > 1000000000LL ? p.timeout_ns : 1000000000LL);
                }
        }
    } else {
        const int w = warp - 1;       // 16-key slice of each tile
        const int gr = lane >> 2;     // fragment row (query head within the group)
        const int tq = lane & 3;      // fragment column pair
        // Q as the A operand (rows = heads of the group, zero beyond G), k-steps of 16 d
        uint32_t qa[4][4];
        float qscale_inv = 1.f;
        {
            const __nv_bfloat16 *qb = p.q + ((size_t)b * p.Hq + (size_t)g * p.G) * kD;
            auto qpair = [&](int row, int d) -> uint32_t {
                if (row >= p.G) return 0u;
                return *reinterpret_cast<const uint32_t *>(qb + (size_t)row * kD + d);
            };
            if (!kFp8) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    qa[kk][0] = qpair(gr, 16 * kk + 2 * tq);
                    qa[kk][1] = qpair(gr + 8, 16 * kk + 2 * tq);
                    qa[kk][2] = qpair(gr, 16 * kk + 8 + 2 * tq);
                    qa[kk][3] = qpair(gr + 8, 16 * kk + 8 + 2 * tq);
                }
            } else {
                // e4m3 caches: f16 MMAs (every e4m3 value is an f16).  q goes to f16
                // times 2^e, the power of two that puts max|q| of the group in
                // [2^14, 2^15), so no element overflows; 2^-e joins the logit scale.
                // The head dimension is visited in the order that lets a lane take
                // K's fragments from 16 consecutive bytes of a key row: in k-step
                // kk, fragment columns 2t, 2t+1 (8+2t, 9+2t) are dimensions
                // 16t + 4kk + 0, 1 (2, 3); q and k use the same order.
                uint32_t raw[4][4];
                float amax = 0.f;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int d0 = 16 * tq + 4 * kk;
                    raw[kk][0] = qpair(gr, d0);
                    raw[kk][1] = qpair(gr + 8, d0);
                    raw[kk][2] = qpair(gr, d0 + 2);
                    raw[kk][3] = qpair(gr + 8, d0 + 2);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&raw[kk][u]);
                        amax = fmaxf(amax, fmaxf(fabsf(__low2float(h)), fabsf(__high2float(h))));
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                const int e = amax > 0.f ? 141 - (int)((__float_as_uint(amax) >> 23) & 0xffu) : 0;
                const int ec = max(-100, min(100, e));
                const float qsc = __uint_as_float((uint32_t)(ec + 127) << 23);
                qscale_inv = __uint_as_float((uint32_t)(127 - ec) << 23);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&raw[kk][u]);
                        qa[kk][u] = pack_f16x2(__low2float(h) * qsc, __high2float(h) * qsc);
                    }
            }
        }
        // e4m3 caches: K's scale (and q's power of two) fold into the logit
        // scale, V's scale into the output
        const float C = kFp8 ? p.c_log2 * p.k_scale[g] * qscale_inv : p.c_log2;
        const uint32_t sbase = smem_u32(smem);
        for (int j = 0; j < n_tiles && ok; ++j) {
            const int st = j % kNS;
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&full[st], (j / kNS) & 1u, abort_flag, p.status, p.timeout_ns))) {
                ok = false;
                break;
            }
            const uint32_t kt = sbase + st * L::kStageBytes;
            uint32_t vt = kt + L::kTileBytes;
            int rw = 16 * w;  // first row of this warp's 16 keys in the tile it reads
            uint4 k8r[L::kSlices][2];  // e4m3 only: this lane's 16 bytes of key row (16w + 64 sl + 8nt + gr)
            if (kFp8) {
                // this warp's keys (16w + 64 sl .. + 15 for each slice sl): K's
                // fragments straight from the e4m3 tile, V widened to f16 into the
                // warp's own staging (the layout the transposing ldmatrix reads);
                // then the raw stage is free again
                const uint8_t *k8 = smem + st * L::kStageBytes;
                const uint8_t *v8 = k8 + L::kTileBytes;
                uint8_t *vs = smem + L::kOffStaging + w * L::kWarpStaging;
#pragma unroll
                for (int sl = 0; sl < L::kSlices; ++sl)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
                        k8r[sl][nt] = *reinterpret_cast<const uint4 *>(
                            k8 + (64 * sl + 16 * w + 8 * nt + gr) * L::kRowBytes + 16 * tq);
#pragma unroll
                for (int it = 0; it < 2 * L::kSlices; ++it) {
                    const int i = lane + 32 * it;
                    const int row = i >> 2, ch = i & 3;  // 16 rows per slice x 4 chunks of 16 values
                    const int trow_ = 64 * (row >> 4) + 16 * w + (row & 15);
                    uint4 lo, hi;
                    e4m3x16_to_f16(*reinterpret_cast<const uint4 *>(v8 + trow_ * L::kRowBytes + ch * 16), lo, hi);
                    *reinterpret_cast<uint4 *>(vs + swz(row, 2 * ch)) = lo;
                    *reinterpret_cast<uint4 *>(vs + swz(row, 2 * ch + 1)) = hi;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
                vt = smem_u32(vs);
                rw = 0;
            }
#pragma unroll
            for (int sl = 0; sl < L::kSlices; ++sl) {
            const int key0 = kbeg + j * kT + 64 * sl + 16 * w;  // first key of this warp's slice
            // ---- S = Q K^T for 16 keys: two n-tiles of 8 keys
            float s[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
                if (kFp8) {
                    const uint32_t w4[4] = {k8r[sl][nt].x, k8r[sl][nt].y, k8r[sl][nt].z, k8r[sl][nt].w};
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma16816_f16(s[nt], qa[kk], e4m3x2_to_f16x2(w4[kk]), e4m3x2_to_f16x2(w4[kk] >> 16));
                } else {
                    const int krow = rw + 8 * nt + (lane & 7);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t b0, b1, b2, b3;  // d chunks 4*half + 0..3
                        ldsm_x4(kt + swz(krow, 4 * half + (lane >> 3)), b0, b1, b2, b3);
                        mma16816(s[nt], qa[2 * half], b0, b1);
                        mma16816(s[nt], qa[2 * half + 1], b2, b3);
                    }
                }
            }
            // ---- mask keys outside [lo, kend); log2-domain logits
            float x[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = key0 + 8 * nt + 2 * tq + (e & 1);
                    x[nt][e] = (key < kend && key >= lo) ? s[nt][e] * C : -INFINITY;
                }
            // ---- online softmax, row gr (elements 0,1) and row gr+8 (elements 2,3)
            float mx_a = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
            const float mn_a = fmaxf(m_a, mx_a);
            const float al_a = (m_a == -INFINITY) ? 0.f : ex2(m_a - mn_a);
            const float sub_a = (mn_a == -INFINITY) ? 0.f : mn_a;
            m_a = mn_a;
            float pv[2][4];
            pv[0][0] = ex2(x[0][0] - sub_a);
            pv[0][1] = ex2(x[0][1] - sub_a);
            pv[1][0] = ex2(x[1][0] - sub_a);
            pv[1][1] = ex2(x[1][1] - sub_a);
            l_a = l_a * al_a + (pv[0][0] + pv[0][1]) + (pv[1][0] + pv[1][1]);
            float al_b = 1.f;
            if (kRows16) {
                float mx_b = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
                const float mn_b = fmaxf(m_b, mx_b);
                al_b = (m_b == -INFINITY) ? 0.f : ex2(m_b - mn_b);
                const float sub_b = (mn_b == -INFINITY) ? 0.f : mn_b;
                m_b = mn_b;
                pv[0][2] = ex2(x[0][2] - sub_b);
                pv[0][3] = ex2(x[0][3] - sub_b);
                pv[1][2] = ex2(x[1][2] - sub_b);
                pv[1][3] = ex2(x[1][3] - sub_b);
                l_b = l_b * al_b + (pv[0][2] + pv[0][3]) + (pv[1][2] + pv[1][3]);
            } else {
                pv[0][2] = pv[0][3] = pv[1][2] = pv[1][3] = 0.f;
            }
#pragma unroll
            for (int jn = 0; jn < 8; ++jn) {
                o[jn][0] *= al_a;
                o[jn][1] *= al_a;
                o[jn][2] *= al_b;
                o[jn][3] *= al_b;
            }
            // ---- O += P V: P from the score accumulators, V via transposing ldmatrix
            uint32_t pa[4];
            if (kFp8) {
                pa[0] = pack_f16x2(pv[0][0], pv[0][1]);
                pa[1] = pack_f16x2(pv[0][2], pv[0][3]);
                pa[2] = pack_f16x2(pv[1][0], pv[1][1]);
                pa[3] = pack_f16x2(pv[1][2], pv[1][3]);
            } else {
                pa[0] = pack_bf16x2(pv[0][0], pv[0][1]);
                pa[1] = pack_bf16x2(pv[0][2], pv[0][3]);
                pa[2] = pack_bf16x2(pv[1][0], pv[1][1]);
                pa[3] = pack_bf16x2(pv[1][2], pv[1][3]);
            }
            // rows of V outside [lo, kend) are zeroed in the operand (cache rows
            // beyond the sequence may hold anything)
            const bool tail = __any_sync(0xffffffffu, key0 + 15 >= kend || key0 < lo);
            const int vrow = rw + 16 * sl + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
            for (int jn = 0; jn < 8; jn += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vt + swz(vrow, jn + (lane >> 4)), b0, b1, b2, b3);
                if (tail) {
                    // b0/b2: keys 2tq, 2tq+1 of the slice; b1/b3: keys 8 + 2tq, 8 + 2tq + 1
                    const int k0 = key0 + 2 * tq, k8 = k0 + 8;
                    auto in = [&](int k) { return k < kend && k >= lo; };
                    const uint32_t m0 = (in(k0) ? 0x0000FFFFu : 0u) | (in(k0 + 1) ? 0xFFFF0000u : 0u);
                    const uint32_t m8 = (in(k8) ? 0x0000FFFFu : 0u) | (in(k8 + 1) ? 0xFFFF0000u : 0u);
                    b0 &= m0;
                    b2 &= m0;
                    b1 &= m8;
                    b3 &= m8;
                }
                if (kFp8) {
                    mma16816_f16(o[jn], pa, b0, b1);
                    mma16816_f16(o[jn + 1], pa, b2, b3);
                } else {
                    mma16816(o[jn], pa, b0, b1);
                    mma16816(o[jn + 1], pa, b2, b3);
                }
            }
            }  // slices
            __syncwarp();
            if (!kFp8 && lane == 0) mbar_arrive(&empty[st]);
        }
        // row sums over the 4 lanes of a fragment row
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    }

    // ---- combine the four consumer warps (ring buffers are idle now)
    __syncthreads();
    if (*abort_flag) return;
    float *red = reinterpret_cast<float *>(smem);  // [4 warps][16 rows][66]: o[64], m, l
    if (warp > 0) {
        const int w = warp - 1, gr = lane >> 2, tq = lane & 3;
        float *ra = red + ((size_t)w * 16 + gr) * 66;
        float *rb = red + ((size_t)w * 16 + gr + 8) * 66;
#pragma unroll
        for (int jn = 0; jn < 8; ++jn) {
            ra[8 * jn + 2 * tq] = o[jn][0];
            ra[8 * jn + 2 * tq + 1] = o[jn][1];
            rb[8 * jn + 2 * tq] = o[jn][2];
            rb[8 * jn + 2 * tq + 1] = o[jn][3];
        }
        if (tq == 0) {
            ra[64] = m_a;
            ra[65] = l_a;
            rb[64] = m_b;
            rb[65] = l_b;
        }
    }
    __syncthreads();
    const int rows = kRows16 ? 16 : 8;
    const float vsc = kFp8 ? p.v_scale[g] : 1.f;  // e4m3 caches: V's dequantisation scale
    for (int e = threadIdx.x; e < rows * kD; e += kThreads) {
        const int r = e / kD, d = e % kD;
        if (r >= p.G) continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, red[((size_t)w * 16 + r) * 66 + 64]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float *rr = red + ((size_t)w * 16 + r) * 66;
            const float f = (rr[64] == -INFINITY) ? 0.f : ex2(rr[64] - M);
            L += f * rr[65];
            O += f * rr[d];
        }
        const int h = g * p.G + r;
        if (nsplit == 1) {
            // the only split of this sequence: the sink joins here, once
            const float sk = p.sinks[h] * kLog2e;
            const float M2 = fmaxf(M, sk);
            const float fo = (M == -INFINITY) ? 0.f : ex2(M - M2);
            const float fs = (sk == -INFINITY) ? 0.f : ex2(sk - M2);
            const float Lt = L * fo + fs;
            const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
            p.out[((size_t)b * p.Hq + h) * kD + d] = __float2bfloat16_rn(O * vsc * fo * inv);
            if (d == 0) p.lse[(size_t)b * p.Hq + h] = Lt > 0.f ? (M2 + log2f(Lt)) * kLn2 : -INFINITY;
        } else {
            const size_t slot = ((size_t)b * p.Hq + h) * p.splits + c;
            p.ws_o[slot * kD + d] = O * vsc;
            if (d == 0) {
                p.ws_ml[slot * 2 + 0] = M;
                p.ws_ml[slot * 2 + 1] = L;
            }
        }
    }
}

// The kernel entry points: the default register allocation, and one held to
// four CTAs per SM (at most 102 registers per thread) for the short e4m3
// splits, whose two-stage ring then fits four CTAs per SM.
template <bool kRows16, bool kPaged, bool kFp8, int kStages>
__global__ void __launch_bounds__(kThreads)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DecodeParams p)
{
    decode_tc_body<kRows16, kPaged, kFp8, kStages>(tmK, tmV, p);
}

template <bool kRows16, bool kPaged, bool kFp8, int kStages>
__global__ void __launch_bounds__(kThreads, 4)
    decode_tc_kernel_4(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const DecodeParams p)
{
    decode_tc_body<kRows16, kPaged, kFp8, kStages>(tmK, tmV, p);
}

}  // namespace

bool decode_bf16_supported(const DecodeShape &s)
{
    const int G = s.Hq / s.Hkv;
    return s.D == kD && G >= 1 && G <= 16 && s.Hq % s.Hkv == 0 && s.splits <= 65535 && s.Hkv <= 65535 &&
           s.B <= 65535;
}

cudaError_t launch_decode_bf16(const void *q, const void *kc, const void *vc, const int *seqlens,
                               const float *sinks, void *out, float *lse, const DecodeShape &s, float *ws_o,
                               float *ws_ml, cudaStream_t st, const float *k_scale, const float *v_scale)
{
    const bool fp8 = k_scale != nullptr;
    DecodeParams p;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.sh = s;
    const int kT = fp8 ? DecLayout<true, ATTN_SINK_DEC_FP8_STAGES>::kT : DecLayout<false, 4>::kT;
    p.box_rows = s.page_size > 0 && s.page_size < kT ? s.page_size : kT;
    p.B = s.B;
    p.Lmax = s.Lmax;
    p.Hq = s.Hq;
    p.Hkv = s.Hkv;
    p.G = s.Hq / s.Hkv;
    p.window = s.window;
    p.splits = s.splits;
    p.chunk = s.chunk;
    p.c_log2 = s.scale * kLog2e;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.seqlens = seqlens;
    p.sinks = sinks;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.ws_o = ws_o;
    p.ws_ml = ws_ml;
    p.status = device_status_ptr();
    p.timeout_ns = wait_timeout_ns();
    const bool paged = s.page_size > 0;
    alignas(64) CUtensorMap mk, mv;
    // contiguous: [B][Lmax][Hkv][64]; paged pool: [num_pages][page_size][Hkv][64]
    const uint64_t rows = paged ? (uint64_t)s.page_size : (uint64_t)s.Lmax;
    const uint64_t outer = paged ? (uint64_t)s.num_pages : (uint64_t)s.B;
    // bf16 rows of 128 bytes (128-byte swizzle, the layout ldmatrix reads);
    // e4m3 rows of 64 bytes, unswizzled (converted by the consumer warps)
    const int eb = fp8 ? 1 : 2;
    const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.Hkv, rows, outer};
    const uint64_t strides[3] = {(uint64_t)kD * eb, (uint64_t)s.Hkv * kD * eb, rows * s.Hkv * kD * eb};
    const uint32_t box[4] = {(uint32_t)kD, 1u, (uint32_t)p.box_rows, 1u};
    if (!encode_tensor_map_4d(&mk, const_cast<void *>(kc), eb, dims, strides, box, !fp8) ||
        !encode_tensor_map_4d(&mv, const_cast<void *>(vc), eb, dims, strides, box, !fp8))
        return cudaErrorInvalidValue;
    const dim3 grid(s.splits, s.Hkv, s.B);
    auto launch = [&](auto kern, int smem_bytes) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem_bytes, st>>>(mk, mv, p);
        return cudaGetLastError();
    };
    constexpr int kF8S = ATTN_SINK_DEC_FP8_STAGES;
    if (fp8) {
        if (paged) return cudaErrorInvalidValue;  // e4m3 caches are contiguous only
        // a split of at most 256 keys (two or three 128-key tiles): two stages
        // and at most 102 registers per thread, so four CTAs share an SM
        auto pick8 = [&](auto stages) -> cudaError_t {
            constexpr int kS = decltype(stages)::value;
            constexpr int s8 = DecLayout<true, kS>::kSmemBytes;
            if constexpr (kS == 2)
                return p.G > 8 ? launch(decode_tc_kernel_4<true, false, true, 2>, s8)
                               : launch(decode_tc_kernel_4<false, false, true, 2>, s8);
            else
                return p.G > 8 ? launch(decode_tc_kernel<true, false, true, kS>, s8)
                               : launch(decode_tc_kernel<false, false, true, kS>, s8);
        };
        return s.chunk <= 256 ? pick8(std::integral_constant<int, 2>{}) : pick8(std::integral_constant<int, kF8S>{});
    }
    // a split of at most 192 keys (a window of 128: 128 keys anywhere, or
    // three whole tiles of a paged cache) needs about three 64-key tiles:
    // three stages hold them, and the smaller ring lets four CTAs share an SM
    // (measured on the window-128 decode of 64 sequences: 17.2 -> 15.4 us;
    // long contiguous splits keep four stages, 336.6 vs 338.8 us dense).  A
    // paged cache moves its tiles in page-sized boxes, and more CTAs per SM
    // keep more of them in flight: three stages there too (dense decode over
    // 16-key pages 388 -> 379 us).
    auto pick = [&](auto stages) -> cudaError_t {
        constexpr int kS = decltype(stages)::value;
        constexpr int sb = DecLayout<false, kS>::kSmemBytes;
        if (p.G > 8)
            return paged ? launch(decode_tc_kernel<true, true, false, kS>, sb)
                         : launch(decode_tc_kernel<true, false, false, kS>, sb);
        return paged ? launch(decode_tc_kernel<false, true, false, kS>, sb)
                     : launch(decode_tc_kernel<false, false, false, kS>, sb);
    };
    return (s.chunk <= 192 || paged) ? pick(std::integral_constant<int, 3>{}) : pick(std::integral_constant<int, 4>{});
}

}  // namespace attn_sink
