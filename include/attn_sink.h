/*
 * attn_sink.h -- C ABI of libattn_sink.so: grouped-query attention whose
 * softmax carries a learned per-head sink logit, on NVIDIA B200 (sm_100a).
 *
 * The operation ("GPT-OSS on day 0", Perplexity, sections "Attention: GQA
 * with Attention Sinks" and "Sink Attention"): every query head h owns a
 * sink logit sink_h that joins the softmax denominator but carries no value
 * row.  For query row i and the keys j it may see,
 *
 *     s_ij  = scale * <q_i, k_j>
 *     M_i   = max(sink_h, max_j s_ij)
 *     Z_i   = exp(sink_h - M_i) + sum_j exp(s_ij - M_i)
 *     out_i = sum_j exp(s_ij - M_i) v_j / Z_i
 *     lse_i = M_i + ln Z_i                        (the sink term included)
 *
 * The sink is a raw logit: it is not multiplied by `scale`.  Query head h
 * reads KV head h / (Hq / Hkv) (grouped-query attention, "GPT-OSS 20B
 * Egitimi: Unsloth, A100 ve Hopper Uyumlulugu", section 1).  Layers are
 * either dense causal (window <= 0) or causal and banded to the last
 * `window` keys (window = 128 in gpt-oss: "GPT-OSS-120B 4-bit ...",
 * section 3).  Query row i of Lq sits at absolute position
 * p_i = i + (Lk - Lq); key j is visible iff j <= p_i and, when window > 0,
 * j > p_i - window.  A row with no visible key gets out = 0 and
 * lse = sink_h (lse = -inf, out = 0 when sink_h = -inf as well).
 *
 * Conventions shared by every call below.
 *   Pointers      device memory owned by the caller, except where a
 *                 parameter says "host".  The library never allocates,
 *                 frees or retains any of them.  Every tensor pointer must be
 *                 16-byte aligned.
 *   dtype         element type of q/k/v/out/dout/dq/dk/dv/caches:
 *                 ATTN_SINK_DTYPE_F32 (exact fp32 CUDA-core path) or
 *                 ATTN_SINK_DTYPE_BF16 (tensor-core path, fp32 accumulation).
 *                 sinks, dsinks and lse are always fp32.
 *   D             head dimension; only 64 is supported.
 *   stream        a cudaStream_t (NULL = legacy default stream).  Calls are
 *                 asynchronous: they enqueue kernels on `stream` and return.
 *   Return value  ATTN_SINK_OK (0) or a negative attn_sink_status.  On a
 *                 non-zero return nothing has been enqueued, except for
 *                 ATTN_SINK_ERR_CUDA, which reports a failed launch.
 *   Timeouts      every device-side wait is bounded; a wait that expires sets
 *                 a per-device status word, and the kernel winds down without
 *                 trapping.  attn_sink_get_device_status() reports it.
 *   Threads       the library keeps no state between calls apart from a
 *                 one-time per-device set-up (kernel attributes, the device
 *                 check), so calls from several host threads are safe.
 */
#ifndef ATTN_SINK_H
#define ATTN_SINK_H

#include <stddef.h>

#if defined(__GNUC__)
#define ATTN_SINK_API __attribute__((visibility("default")))
#else
#define ATTN_SINK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum attn_sink_status {
    ATTN_SINK_OK = 0,
    ATTN_SINK_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, Hq % Hkv != 0, ... */
    ATTN_SINK_ERR_UNSUPPORTED = -2,   /* D != 64, unknown dtype, group size not supported */
    ATTN_SINK_ERR_MISALIGNED = -3,    /* a tensor pointer is not 16-byte aligned */
    ATTN_SINK_ERR_ARCH = -4,          /* the current device is not sm_100 (B200) */
    ATTN_SINK_ERR_WORKSPACE = -5,     /* workspace missing or smaller than required */
    ATTN_SINK_ERR_CUDA = -6,          /* a CUDA runtime/driver call or launch failed */
    ATTN_SINK_ERR_TIMEOUT = -7,       /* a bounded device-side wait expired */
    ATTN_SINK_ERR_NO_DEVICE = -8,     /* no CUDA device is visible */
    ATTN_SINK_ERR_SCRATCH_LIMIT = -9  /* attn_sink_decode_noalloc: the problem needs more
                                         scratch than ATTN_SINK_NOALLOC_SCRATCH_BYTES */
} attn_sink_status;

enum { ATTN_SINK_DTYPE_F32 = 0, ATTN_SINK_DTYPE_BF16 = 1 };

/*
 * Prefill forward ("GPT-OSS on day 0", section "Sink Attention": the sink
 * seeds the running maximum of the online softmax).
 *   q     [B, Lq, Hq, D]   k, v [B, Lk, Hkv, D]   (dtype)
 *   sinks [Hq] fp32
 *   out   [B, Lq, Hq, D]   (dtype, written)
 *   lse   [B, Hq, Lq] fp32 (written; natural log, sink included)
 *   window <= 0: dense causal; window > 0: causal band of `window` keys.
 *   scale: multiplies <q, k> (usually 1/sqrt(D)); for dtype BF16 it must be
 *          positive and finite (ATTN_SINK_ERR_UNSUPPORTED otherwise).
 * Lq > Lk is allowed (leading rows then see no key).  B*Lq*Hq*D and
 * B*Lk*Hkv*D must stay below 2^31 elements per tensor for dtype F32.
 * For dtype BF16 the kernel's CTAs share out the work among themselves
 * through the hardware's cluster launch control (a running CTA takes over
 * the work of a CTA of the same launch that has not started); no state is
 * kept between launches, so any number of launches may run at once, on any
 * streams, and launches captured in a CUDA graph may be replayed.
 */
ATTN_SINK_API int attn_sink_fwd(const void *q, const void *k, const void *v, const float *sinks,
                  void *out, float *lse, int B, int Lq, int Lk, int Hq, int Hkv, int D,
                  int window, float scale, int dtype, void *stream);

/*
 * The bf16 prefill forward of attn_sink_fwd with every tensor in HOST memory:
 * q, k, v, sinks are read from host memory and out, lse written back to it,
 * with the transfers overlapped with the computation.  The query positions
 * are cut into up to `n_chunks` chunks (1..64; multiples of 128 positions;
 * with three or more, the first and the last hold half as many positions as
 * the others, since nothing overlaps their copies): chunk c's
 * rows need only the keys up to its last position, so while chunk c is
 * computed, chunk c + 1's q rows and new k, v rows travel to the device and
 * chunk c - 1's out rows travel back (lse once, at the end; host-to-device and
 * device-to-host copies run on two streams of the library's own, the kernels
 * on `stream`; the call returns once everything is enqueued, and `stream` is
 * ordered after the last copy, so synchronising `stream` waits for the whole
 * call).  Each row's arithmetic is that of attn_sink_fwd on the same inputs
 * (the chunks hold whole work items of the forward, so the same tiles), so
 * the results are bit-for-bit identical.
 *   q_host [B, Lq, Hq, D], k_host, v_host [B, Lk, Hkv, D] bf16; sinks_host
 *   [Hq] fp32; out_host [B, Lq, Hq, D] bf16 and lse_host [B, Hq, Lq] fp32
 *   (written).  Host buffers should be page-locked (cudaHostAlloc, or
 *   torch's pin_memory) for the copies to overlap; pageable memory gives the
 *   same results without the overlap.  The caller keeps them alive and
 *   unchanged until `stream` has passed the call.
 *   workspace: device memory of attn_sink_fwd_host_workspace_size() bytes,
 *   16-byte aligned, owned by the caller (the device copies of q, k, v,
 *   sinks, out and lse); it must not be in use by other work on other
 *   streams during the call.
 *   Lq <= Lk (else ATTN_SINK_ERR_UNSUPPORTED); other arguments and errors as
 *   for attn_sink_fwd with dtype BF16; ATTN_SINK_ERR_INVALID_ARG for
 *   n_chunks outside 1..64.
 */
ATTN_SINK_API size_t attn_sink_fwd_host_workspace_size(int B, int Lq, int Lk, int Hq, int Hkv, int D);
ATTN_SINK_API int attn_sink_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                  const float *sinks_host, void *out_host, float *lse_host, int B, int Lq, int Lk,
                  int Hq, int Hkv, int D, int window, float scale, int n_chunks,
                  void *workspace, size_t ws_bytes, void *stream);

/*
 * Prefill forward over packed ragged sequences ("varlen"): a batch of B
 * sequences of different lengths stored back to back, as a prefill server
 * that gathers requests of any length receives them (the pages separate the
 * prefill of requests from their decode -- "GPT-OSS on day 0", section "Cost
 * i rendiment" -- and measure prefill over batches of mixed sizes).  Each
 * sequence is an independent problem with the operation of attn_sink_fwd.
 *   q, out [total_q, Hq, D] bf16     k, v [total_k, Hkv, D] bf16
 *   cu_seqlens_q, cu_seqlens_k [B + 1] int32, device: sequence b owns query
 *           rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key rows
 *           [cu_seqlens_k[b], cu_seqlens_k[b+1]); its query i sits at
 *           position i + (Lk_b - Lq_b) (bottom-right causal alignment, so a
 *           sequence with a cached prefix has Lk_b > Lq_b).  Offsets must be
 *           non-decreasing from 0; they are clamped into [0, total] on the
 *           device, so no bad offset reads or writes out of bounds.
 *   max_seqlen_q  host-side upper bound on every Lq_b (rows past it are not
 *           computed).  A sequence may be empty.
 *   lse     [Hq, total_q] fp32 (natural log, sink included).
 *   sinks, window, scale: as attn_sink_fwd (scale positive and finite).
 * bf16 only.  Errors: INVALID_ARG for null pointers or non-positive sizes,
 * otherwise as attn_sink_fwd.  Nothing is allocated; asynchronous on stream.
 */
ATTN_SINK_API int attn_sink_fwd_varlen(const void *q, const void *k, const void *v, const float *sinks,
                  void *out, float *lse, const int *cu_seqlens_q, const int *cu_seqlens_k,
                  int B, int max_seqlen_q, int total_q, int total_k, int Hq, int Hkv, int D,
                  int window, float scale, void *stream);

/*
 * Prefill forward with q, k and v in FP8 (e4m3): the operation of
 * attn_sink_fwd with q, k and v read at one byte per element.  The pages
 * serve gpt-oss at FP8 precision ("GPT-OSS on day 0", section "GPT-OSS a
 * Hopper"); the format and its scale granularity are not given there: here
 * every query head has one fp32 scale for q and every KV head one for k and
 * one for v (the value of an element is code * its head's scale).
 *   q        [B, Lq, Hq, D] e4m3 codes     k, v [B, Lk, Hkv, D] e4m3 codes
 *            (OCP FP8 E4M3: bias 7, 3 mantissa bits, subnormals, 0x7f / 0xff
 *            NaN; NaN codes in the inputs give NaN outputs)
 *   q_scale  [Hq] fp32, k_scale, v_scale [Hkv] fp32, device; positive and
 *            finite (the kernel takes the row maximum of the raw products)
 *   sinks, window, scale: as attn_sink_fwd (scale positive and finite)
 *   out      [B, Lq, Hq, D] bf16          lse [B, Hq, Lq] fp32
 *   workspace device memory of attn_sink_fwd_fp8_workspace_size(B, Lk, Hkv, D)
 *            bytes (v widened to f16), 16-byte aligned, owned by the caller;
 *            its contents on return are unspecified.
 * Q K^T runs on the 8-bit tensor-core path: the products of e4m3 values are
 * exact and accumulate in fp32; the scales then multiply the logits.  V is
 * widened exactly to f16 (one pass into the workspace) and P (in f16) times V
 * runs on the 16-bit path, so the result carries the rounding of the bf16
 * forward, not of FP8 attention probabilities.  Fixed-length batches only.
 * Errors as attn_sink_fwd, INVALID_ARG for a null scale pointer, WORKSPACE
 * for a missing or short workspace.  Nothing is allocated; asynchronous on
 * stream.
 */
ATTN_SINK_API int attn_sink_fwd_fp8(const void *q, const void *k, const void *v, const float *q_scale,
                  const float *k_scale, const float *v_scale, const float *sinks, void *out,
                  float *lse, int B, int Lq, int Lk, int Hq, int Hkv, int D, int window,
                  float scale, void *workspace, size_t ws_bytes, void *stream);

/* Bytes of workspace attn_sink_fwd_fp8 needs (B * Lk * Hkv * D * 2; 0 for a non-positive size). */
ATTN_SINK_API size_t attn_sink_fwd_fp8_workspace_size(int B, int Lk, int Hkv, int D);

/*
 * QKV prologue: the step just before attention, in one pass over the QKV
 * projection's output.  The pages give gpt-oss QKV projections with biases
 * and YaRN rotary position encoding "as in DeepSeek-V3" ("GPT-OSS on day 0",
 * section "Attention: GQA with Attention Sinks"), extended to 131072 tokens
 * ("GPT-OSS-120B 4-bit ...", section 3); they give no parameter values, so
 * the rotation's parameters are arguments.  For token t at position p:
 *   y = qkv[t] + bias (fp32), split into q (Hq heads), k (Hkv), v (Hkv);
 *   q and k are rotated pair by pair, with rotary frequency f_i =
 *   rope_theta^(-2i/D) for pair i of D/2, corrected by YaRN when
 *   rope_factor > 1: with d(n) = D ln(L0 / (2 pi n)) / (2 ln rope_theta),
 *   L0 = rope_original_max_pos, the weight e_i = 1 - clamp((i - d(beta_fast))
 *   / (d(beta_slow) - d(beta_fast)), 0, 1) keeps f_i where a wavelength fits
 *   many times into L0 and interpolates to f_i / rope_factor where it does
 *   not: f'_i = e_i f_i + (1 - e_i) f_i / rope_factor; cos and sin of
 *   p f'_i are scaled by the attention factor 0.1 ln(rope_factor) + 1.
 *   Pair i is (i, i + D/2) (interleaved = 0) or (2i, 2i + 1) (interleaved = 1);
 *   (x, y) -> (x cos - y sin, y cos + x sin).  v gets its bias only.
 *   rope_factor <= 1 is plain rotary embedding (no correction, factor 1).
 *   qkv     [T, (Hq + 2 Hkv) * D] bf16, q columns first, then k, then v
 *   bias    [(Hq + 2 Hkv) * D] fp32, or NULL for none
 *   positions [T] int32, device
 *   kv_rows [T] int32, device, or NULL: token t's k and v go to row
 *           kv_rows[t] (row t) of k_out / v_out, so a decode step can append
 *           them to a cache laid out [B, Lmax, Hkv, D] (row b * Lmax + p) in
 *           the same pass; a row outside [0, kv_rows_total) is not written.
 *   q_out   [T, Hq, D] bf16     k_out, v_out [kv_rows_total, Hkv, D] bf16
 * Angles are formed and reduced in fp64.  D must be 64.  Errors:
 * INVALID_ARG for null pointers, non-positive sizes, kv_rows NULL with
 * kv_rows_total < T, rope_theta <= 1, rope_factor <= 0, or (rope_factor > 1)
 * rope_original_max_pos <= 0 or not beta_fast > beta_slow > 0;
 * UNSUPPORTED for D != 64.  Nothing is allocated; asynchronous on stream.
 */
ATTN_SINK_API int attn_sink_qkv_prologue(const void *qkv, const float *bias, const int *positions,
                  const int *kv_rows, void *q_out, void *k_out, void *v_out, int T, int Hq,
                  int Hkv, int D, int kv_rows_total, float rope_theta, float rope_factor,
                  int rope_original_max_pos, float beta_fast, float beta_slow, int interleaved,
                  void *stream);

/*
 * Split-KV decode over a contiguous per-sequence KV cache with ragged
 * lengths ("GPT-OSS on day 0", section "Sink Attention": attention is split
 * along the KV length as well as across heads, and the sink must be counted
 * once, not once per split).
 *   q        [B, Hq, D]            one query per sequence (dtype)
 *   k_cache, v_cache [B, Lmax, Hkv, D]  (dtype)
 *   seqlens  [B] int32, device     cached length of each sequence, in
 *                                  [1, Lmax]; the query sits at position
 *                                  seqlens[b] - 1 (its own key is already
 *                                  in the cache).  Values outside [1, Lmax]
 *                                  are clamped on the device.
 *   sinks    [Hq] fp32
 *   out      [B, Hq, D] (dtype)    lse [B, Hq] fp32
 *   num_splits  0 = choose automatically, else 1..32: the visible range of
 *               the longest possible sequence is cut into num_splits chunks
 *               of equal length (a multiple of 64 keys); sequence b uses as
 *               many chunks as its own range needs.
 *   workspace   device scratch of at least
 *               attn_sink_decode_workspace_size(B, Hq, D, Lmax, window, num_splits)
 *               bytes (may be NULL when that size is 0).  Its contents on
 *               entry do not matter.
 */
ATTN_SINK_API int attn_sink_decode(const void *q, const void *k_cache, const void *v_cache,
                     const int *seqlens, const float *sinks, void *out, float *lse,
                     int B, int Lmax, int Hq, int Hkv, int D, int window, float scale,
                     int num_splits, void *workspace, size_t ws_bytes, int dtype,
                     void *stream);

/* Bytes of decode workspace for these sizes (0 when a single split suffices). */
ATTN_SINK_API size_t attn_sink_decode_workspace_size(int B, int Hq, int D, int Lmax, int window, int num_splits);

/*
 * Split-KV decode over a KV cache stored in FP8 (e4m3): the operation of
 * attn_sink_decode with the cached keys and values read at one byte per
 * element, half the bytes of a bf16 cache.  The pages serve gpt-oss at FP8
 * precision ("GPT-OSS on day 0", section "GPT-OSS a Hopper") and size the KV
 * cache in proportion to its element size ("How much computing power is
 * required for gpt-oss deployment?", the question on the KV cache and context
 * length); the cache format and its scale granularity are not given there:
 * here every KV head has one fp32 scale for K and one for V.
 *   q        [B, Hq, D] bf16
 *   k_cache, v_cache [B, Lmax, Hkv, D] e4m3 codes (OCP FP8 E4M3: bias 7,
 *            3 mantissa bits, subnormals, no infinities, 0x7f / 0xff NaN);
 *            the key (value) of head g is code * k_scale[g] (* v_scale[g]).
 *   k_scale, v_scale [Hkv] fp32, device.
 *   seqlens, sinks, window, scale, num_splits, workspace: as attn_sink_decode
 *            (the workspace size is attn_sink_decode_workspace_size's).
 *   out      [B, Hq, D] bf16           lse [B, Hq] fp32
 * Each code is widened exactly (e4m3 -> f16) and the scales are applied in
 * fp32: K's to the logits, V's to the output.  Cache rows beyond a sequence's
 * length may hold any bytes, NaN codes included.  Errors as attn_sink_decode;
 * a null scale pointer is INVALID_ARG.
 */
ATTN_SINK_API int attn_sink_decode_fp8(const void *q, const void *k_cache, const void *v_cache,
                     const float *k_scale, const float *v_scale, const int *seqlens,
                     const float *sinks, void *out, float *lse, int B, int Lmax, int Hq, int Hkv,
                     int D, int window, float scale, int num_splits, void *workspace,
                     size_t ws_bytes, void *stream);

/*
 * Split-KV decode over a paged KV cache: the same operation as
 * attn_sink_decode, with each sequence's cached keys and values gathered
 * through a page table instead of one contiguous [Lmax] slab per sequence
 * (the pages name partitioned KV caches as the way to hold long contexts --
 * "How much computing power is required for gpt-oss deployment?", the
 * question on the KV cache and context length -- and split the attention
 * along the KV length -- "GPT-OSS on day 0", section "Sink Attention").
 *   k_pages, v_pages  [num_pages, page_size, Hkv, D] bf16: the page pool
 *   page_table [B, max_pages_per_seq] int32, device: token t of sequence b
 *              sits in slot t % page_size of page
 *              page_table[b][t / page_size].  Only the first
 *              ceil(seqlens[b] / page_size) entries of a row are read; the
 *              rest may hold anything.  Entries outside [0, num_pages) read
 *              zeros (no fault).  Pages may be shared between sequences.
 *   page_size  8, 16, 32 or a multiple of 64.
 *   seqlens    [B] int32 in [1, max_pages_per_seq * page_size] (clamped on
 *              the device), with the query at position seqlens[b] - 1.
 *   q, sinks, out, lse, window, scale, num_splits: as attn_sink_decode.
 *   dtype      ATTN_SINK_DTYPE_BF16 only (F32 returns UNSUPPORTED).
 *   workspace  at least attn_sink_decode_paged_workspace_size(B, Hq, D,
 *              max_pages_per_seq, page_size, window, num_splits) bytes.
 * Errors: INVALID_ARG for a null pointer, a page_size not listed above,
 * non-positive sizes or max_pages_per_seq * page_size >= 2^31; otherwise as
 * attn_sink_decode.  Nothing is allocated; the call is asynchronous on
 * `stream`.
 */
ATTN_SINK_API int attn_sink_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                     const int *page_table, const int *seqlens, const float *sinks, void *out,
                     float *lse, int B, int max_pages_per_seq, int page_size, int num_pages,
                     int Hq, int Hkv, int D, int window, float scale, int num_splits,
                     void *workspace, size_t ws_bytes, int dtype, void *stream);

/* Bytes of paged-decode workspace for these sizes (0 when a single split suffices). */
ATTN_SINK_API size_t attn_sink_decode_paged_workspace_size(int B, int Hq, int D, int max_pages_per_seq,
                     int page_size, int window, int num_splits);

/*
 * Size of the scratch buffer built into the library for
 * attn_sink_decode_noalloc: 32 MiB of device memory, reserved on every GPU
 * that loads the library and held until the process exits.
 */
#define ATTN_SINK_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * attn_sink_decode for callers that cannot allocate device memory.  The
 * pages describe no such call; it exists for users of this library whose
 * device memory is owned by someone else -- a plugin inside an inference
 * server or framework that must not go around the host's allocator, or a
 * latency-critical decode loop where a cudaMalloc (which can synchronise the
 * device, and can fail) is not acceptable -- and who therefore cannot supply
 * the workspace attn_sink_decode needs.
 *
 * Arguments, layouts, results and errors are those of attn_sink_decode,
 * minus the workspace: the split partials go to a file-scope scratch array
 * of ATTN_SINK_NOALLOC_SCRATCH_BYTES inside the library.  Nothing is
 * allocated: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - A problem whose attn_sink_decode_workspace_size(...) exceeds
 *     ATTN_SINK_NOALLOC_SCRATCH_BYTES is rejected with
 *     ATTN_SINK_ERR_SCRATCH_LIMIT before anything is enqueued (pass a
 *     smaller num_splits, or use attn_sink_decode with your own workspace).
 *   - Every call on a device shares that device's one scratch array and the
 *     array keeps the last call's contents.  Calls whose kernels can overlap
 *     on the GPU (different streams without ordering between them) race on
 *     it and give wrong results; order them on one stream or use
 *     attn_sink_decode.  No part of the scratch needs to start at zero: every
 *     partial is written before it is read.
 *   - The first call on a device looks up the array's device address (a
 *     one-time set-up with that device current); make that first call before
 *     any stream capture begins.
 */
ATTN_SINK_API int attn_sink_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                     const int *seqlens, const float *sinks, void *out, float *lse,
                     int B, int Lmax, int Hq, int Hkv, int D, int window, float scale,
                     int num_splits, int dtype, void *stream);

/*
 * Backward of attn_sink_fwd, derived from the definition above (the pages
 * give no gradient).  With P_ij = exp(s_ij - lse_i), P_sink_i =
 * exp(sink_h - lse_i) and D_i = <dout_i, out_i>:
 *   dS_ij  = P_ij (<dout_i, v_j> - D_i)
 *   dq_i   = scale * sum_j dS_ij k_j
 *   dk_j   = scale * sum over (query heads of j's group, rows i) dS_ij q_i
 *   dv_j   = sum over (query heads of j's group, rows i) P_ij dout_i
 *   dsinks_h = - sum over (b, i) P_sink_i D_i
 * Inputs: q, k, v, sinks as for attn_sink_fwd; out and lse as written by
 * attn_sink_fwd for the same arguments; dout [B, Lq, Hq, D] (dtype).
 * Outputs (overwritten, not accumulated): dq [B, Lq, Hq, D],
 * dk, dv [B, Lk, Hkv, D] (dtype); dsinks [Hq] fp32, summed over the batch.
 * Determinism: dk, dv and dsinks are identical run to run, and so is dq for
 * dtype F32.  For dtype BF16, dq is summed over 128-key tiles by fp32 atomic
 * adds in L2 (a TMA reduce-add), so its fp32 sum -- and rarely its bf16
 * rounding -- may differ in the last bit between runs.
 *   workspace  device scratch of at least
 *              attn_sink_bwd_workspace_size(B, Lq, Lk, Hq, Hkv, D, dtype)
 *              bytes (for BF16 it holds an fp32 copy of dq); contents on
 *              entry do not matter.
 */
ATTN_SINK_API int attn_sink_bwd(const void *q, const void *k, const void *v, const float *sinks,
                  const void *out, const void *dout, const float *lse,
                  void *dq, void *dk, void *dv, float *dsinks,
                  int B, int Lq, int Lk, int Hq, int Hkv, int D, int window, float scale,
                  void *workspace, size_t ws_bytes, int dtype, void *stream);

ATTN_SINK_API size_t attn_sink_bwd_workspace_size(int B, int Lq, int Lk, int Hq, int Hkv, int D, int dtype);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word.  Returns ATTN_SINK_OK, ATTN_SINK_ERR_TIMEOUT if a bounded device
 * wait expired since the last call, or ATTN_SINK_ERR_CUDA if the
 * synchronisation itself failed.
 */
ATTN_SINK_API int attn_sink_get_device_status(void *stream);

/*
 * Upper bound, in nanoseconds, on any single device-side wait in kernels
 * launched after this call (default 2e9, i.e. 2 s; values <= 0 restore the
 * default).  Process-wide.  Returns the previous value.
 */
ATTN_SINK_API long long attn_sink_set_wait_timeout_ns(long long ns);

/* Static description of a status code. */
ATTN_SINK_API const char *attn_sink_strerror(int status);

/*
 * The cudaError_t value behind the most recent ATTN_SINK_ERR_CUDA returned to
 * the calling host thread (0 if none).  Not cleared by later successful calls.
 */
ATTN_SINK_API int attn_sink_last_cuda_error(void);

/* Library version as 10000*major + 100*minor + patch. */
ATTN_SINK_API int attn_sink_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_SINK_H */
