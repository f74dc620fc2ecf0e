// kernels.h -- internal launch interface between the C ABI (attn_sink_api.cu)
// and the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace attn_sink {

// Device status word bits (read back by attn_sink_get_device_status).
enum : unsigned { STATUS_TIMEOUT = 1u };

struct AttnShape {
    int B, Lq, Lk, Hq, Hkv, D, window;
    float scale;
    // packed ragged sequences (varlen): cu_q / cu_k [B + 1] device offsets into
    // q [total_q, Hq, D] and k, v [total_k, Hkv, D]; Lq is then the longest
    // sequence's query count (an upper bound).  nullptr: fixed-length batch.
    const int *cu_q = nullptr, *cu_k = nullptr;
    int total_q = 0, total_k = 0;
    // > 0: lse's stride between heads (B = 1 only), so that a launch over some
    // query positions writes its lse into the columns of a wider [Hq, L] array
    int lse_hs = 0;
};

struct DecodeShape {
    int B, Lmax, Hq, Hkv, D, window;
    float scale;
    int splits;  // maximum number of chunks per sequence
    int chunk;   // keys per chunk (multiple of 64)
    int align;   // 0, or 64: the split range starts at the visible start rounded down to this
    // paged caches (pool [num_pages, page_size, Hkv, D]; page_table [B, max_pages]); 0 = contiguous
    int page_size, max_pages, num_pages;
    const int *page_table;
};

// First key of sequence b's split range and its number of splits (shared by the
// split kernels and the combine kernel).
__host__ __device__ inline void decode_range(const DecodeShape &s, int len, int &lo, int &lo_al, int &nsplit)
{
    lo = s.window > 0 ? (len - s.window > 0 ? len - s.window : 0) : 0;
    lo_al = s.align > 0 ? lo / s.align * s.align : lo;
    nsplit = (len - lo_al + s.chunk - 1) / s.chunk;
}

// Sequence b of a prefill batch: fixed-length sequences (cu == nullptr:
// length fixed_len, its own batch slot) or packed ragged sequences whose rows
// are [cu[b], cu[b + 1]) of one [total, H, D] tensor.  Offsets are clamped
// into [0, total], so any cu array yields in-bounds rows.
struct SeqRows {
    int len;   // rows of the sequence
    int row0;  // its first row in the packed tensor (0 for fixed-length batches)
};
__device__ __forceinline__ SeqRows seq_rows(const int *cu, int b, int fixed_len, int total)
{
    if (cu == nullptr) return {fixed_len, 0};
    const int a = min(max(cu[b], 0), total);
    const int e = min(max(cu[b + 1], a), total);
    return {e - a, a};
}

// Per-device status word (bit STATUS_TIMEOUT set by an expired bounded wait).
unsigned *device_status_ptr();
long long wait_timeout_ns();

// Exact CUDA-core path (T = float or __nv_bfloat16).
template <typename T>
cudaError_t launch_fwd_simt(const T *q, const T *k, const T *v, const float *sinks, T *out, float *lse,
                            const AttnShape &s, cudaStream_t st);
template <typename T>
cudaError_t launch_bwd_simt(const T *q, const T *k, const T *v, const float *sinks, const T *out,
                            const T *dout, const float *lse, T *dq, T *dk, T *dv, float *dsinks,
                            const AttnShape &s, void *ws, cudaStream_t st);
size_t bwd_simt_workspace_bytes(const AttnShape &s);
// row pre-pass of the backward (D_i and the dsink terms; with zero_rows, it
// also clears the fp32 dQ accumulator [B, Lq, Hq, 64])
template <typename T>
cudaError_t launch_bwd_rows(const T *out, const T *dout, const float *lse, const float *sinks, float *Drow,
                            float *terms, float *zero_rows, const AttnShape &s, cudaStream_t st);

// Tensor-core (tcgen05) bf16 backward main pass (+ dQ fp32 accumulation and
// conversion, and the dsink sums of the row pre-pass's terms); dq_acc must
// hold zeros on entry (launch_bwd_rows clears it).
size_t bwd_tc_dq_acc_bytes(const AttnShape &s);
bool bwd_tc_supported(const AttnShape &s);
cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const void *dout, const float *lse,
                          const float *Drow, const float *terms, float *dsinks, float *dq_acc, void *dq, void *dk,
                          void *dv, const AttnShape &s, cudaStream_t st);

template <typename T>
cudaError_t launch_decode_simt(const T *q, const T *kc, const T *vc, const int *seqlens, const float *sinks,
                               T *out, float *lse, const DecodeShape &s, float *ws_o, float *ws_ml,
                               cudaStream_t st);
template <typename T>
cudaError_t launch_decode_combine(const int *seqlens, const float *sinks, T *out, float *lse,
                                  const DecodeShape &s, const float *ws_o, const float *ws_ml, cudaStream_t st);

// Tensor-core bf16 prefill forward of short-window banded layers: one K/V tile
// per work item, exact (single-pass) softmax.
cudaError_t launch_fwd_band(const void *q, const void *k, const void *v, const float *sinks, void *out,
                            float *lse, const AttnShape &s, cudaStream_t st);
bool fwd_band_supported(const AttnShape &s);

// Tensor-core (tcgen05 / TMEM / TMA) bf16 prefill forward.
cudaError_t launch_fwd_tc(const void *q, const void *k, const void *v, const float *sinks, void *out,
                          float *lse, const AttnShape &s, cudaStream_t st);
// e4m3 q, k, v with fp32 scales per query head (q) and per KV head (k, v);
// fixed-length batches; v16 holds fwd_fp8_workspace_bytes (v widened to f16)
size_t fwd_fp8_workspace_bytes(const AttnShape &s);
cudaError_t launch_fwd_tc_fp8(const void *q, const void *k, const void *v, const float *q_scale,
                              const float *k_scale, const float *v_scale, const float *sinks, void *out, float *lse,
                              void *v16, const AttnShape &s, cudaStream_t st);
bool fwd_tc_supported(const AttnShape &s);

// The bf16 prefill forward from and to host memory, chunks of query positions
// overlapping their transfers with the computation (host_fwd.cu); Lq <= Lk.
constexpr int kFwdHostMaxChunks = 64;
size_t fwd_host_workspace_bytes(const AttnShape &s);
cudaError_t run_fwd_host(const void *q_h, const void *k_h, const void *v_h, const float *sinks_h, void *out_h,
                         float *lse_h, const AttnShape &s, int n_chunks, void *workspace, cudaStream_t st);

// bf16 split-KV decode: TMA-staged K/V, tensor-core (mma.sync) group scores.
// With k_scale / v_scale ([Hkv] fp32, device) the caches hold e4m3 values
// whose real values are code * scale of their KV head.
cudaError_t launch_decode_bf16(const void *q, const void *kc, const void *vc, const int *seqlens,
                               const float *sinks, void *out, float *lse, const DecodeShape &s, float *ws_o,
                               float *ws_ml, cudaStream_t st, const float *k_scale = nullptr,
                               const float *v_scale = nullptr);
bool decode_bf16_supported(const DecodeShape &s);

// QKV prologue: bias, YaRN rotary embedding of q and k, split into q / k / v.
struct RopeParams {
    double base, factor, original_max_pos, beta_fast, beta_slow;
    int interleaved;  // 0: pairs (i, i + D/2); 1: pairs (2i, 2i + 1)
};
cudaError_t launch_qkv_prologue(const void *qkv, const float *bias, const int *positions, const int *kv_rows,
                                void *q, void *k, void *v, int T, int Hq, int Hkv, int kv_rows_total,
                                const RopeParams &r, cudaStream_t st);

// Driver entry point for cuTensorMapEncodeTiled (resolved once through the runtime).
bool encode_tensor_map_4d(void *map, void *gaddr, int elem_bytes, const uint64_t dims[4],
                          const uint64_t strides_bytes[3], const uint32_t box[4], bool swizzle128);
// the same with the swizzle span given in bytes (0, 64 or 128)
bool encode_tensor_map_4d_sw(void *map, void *gaddr, int elem_bytes, const uint64_t dims[4],
                             const uint64_t strides_bytes[3], const uint32_t box[4], int swizzle_bytes);

}  // namespace attn_sink
