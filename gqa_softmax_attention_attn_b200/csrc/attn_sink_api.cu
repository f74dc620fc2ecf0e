// attn_sink_api.cu -- the C ABI declared in include/attn_sink.h: argument
// checks, the one-time per-device set-up, and kernel dispatch.  The library
// allocates no device or host memory on any call path.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/attn_sink.h"
#include "kernels.h"

namespace attn_sink {

__device__ unsigned g_device_status = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr long long kDefaultTimeoutNs = 2000000000LL;

std::atomic<long long> g_timeout_ns{kDefaultTimeoutNs};

struct DeviceState {
    std::once_flag once;
    int status = ATTN_SINK_ERR_CUDA;  // result of the set-up
    unsigned *status_ptr = nullptr;
};
DeviceState g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

int current_device(int *dev)
{
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return ATTN_SINK_ERR_NO_DEVICE;
    }
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) {
        cudaGetLastError();
        return ATTN_SINK_ERR_CUDA;
    }
    return ATTN_SINK_OK;
}

// One-time per-device set-up, run with that device current: the device must
// be an sm_100 part (the clean counterpart of a backend that only runs on one
// architecture), and the status word's device address is looked up.
int ensure_device()
{
    int dev = 0;
    int rc = current_device(&dev);
    if (rc != ATTN_SINK_OK) return rc;
    DeviceState &d = g_dev[dev];
    std::call_once(d.once, [&d, dev]() {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
            cudaGetLastError();
            d.status = ATTN_SINK_ERR_CUDA;
            return;
        }
        if (prop.major != 10 || prop.minor != 0) {
            d.status = ATTN_SINK_ERR_ARCH;
            return;
        }
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_device_status) != cudaSuccess) {
            cudaGetLastError();
            d.status = ATTN_SINK_ERR_CUDA;
            return;
        }
        d.status_ptr = static_cast<unsigned *>(ptr);
        d.status = ATTN_SINK_OK;
    });
    return d.status;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int Lq, int Lk, int Hq, int Hkv, int D, int dtype)
{
    if (B <= 0 || Lq <= 0 || Lk <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return ATTN_SINK_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ATTN_SINK_ERR_INVALID_ARG;
    if (D != 64) return ATTN_SINK_ERR_UNSUPPORTED;
    if (dtype != ATTN_SINK_DTYPE_F32 && dtype != ATTN_SINK_DTYPE_BF16) return ATTN_SINK_ERR_UNSUPPORTED;
    if (B > 65535 || Hq > 65535) return ATTN_SINK_ERR_UNSUPPORTED;
    return ATTN_SINK_OK;
}

thread_local int g_last_cuda_error = 0;

int launch_status(cudaError_t e)
{
    if (e == cudaSuccess) return ATTN_SINK_OK;
    g_last_cuda_error = (int)e;
    cudaGetLastError();
    return ATTN_SINK_ERR_CUDA;
}

int auto_splits(int Lmax, int window)
{
    const int lvis = window > 0 ? (window < Lmax ? window : Lmax) : Lmax;
    int s = (lvis + 2047) / 2048;
    if (s < 1) s = 1;
    if (s > 32) s = 32;
    return s;
}

DecodeShape decode_shape(int B, int Lmax, int Hq, int Hkv, int D, int window, float scale, int num_splits)
{
    DecodeShape s{};
    s.B = B;
    s.Lmax = Lmax;
    s.Hq = Hq;
    s.Hkv = Hkv;
    s.D = D;
    s.window = window;
    s.scale = scale;
    const int lvis = window > 0 ? (window < Lmax ? window : Lmax) : Lmax;
    s.splits = num_splits > 0 ? num_splits : auto_splits(Lmax, window);
    int chunk = (lvis + s.splits - 1) / s.splits;
    chunk = (chunk + 63) / 64 * 64;
    s.chunk = chunk;
    // splits that can actually be used by the longest visible range
    s.splits = (lvis + chunk - 1) / chunk;
    return s;
}

// Paged caches: tiles start on multiples of 64 keys, so a banded sequence's
// split range can begin up to 63 keys before its visible start.
bool paged_sizes_ok(int page_size, int max_pages, int num_pages)
{
    if (page_size <= 0 || max_pages <= 0 || num_pages <= 0) return false;
    if (!(page_size % 64 == 0 || page_size == 8 || page_size == 16 || page_size == 32)) return false;
    return (long long)max_pages * page_size <= 0x7fffffffLL;
}

DecodeShape decode_shape_paged(int B, int max_pages, int page_size, int num_pages, const int *page_table, int Hq,
                               int Hkv, int D, int window, float scale, int num_splits)
{
    const int Lmax = max_pages * page_size;
    DecodeShape s{};
    s.B = B;
    s.Lmax = Lmax;
    s.Hq = Hq;
    s.Hkv = Hkv;
    s.D = D;
    s.window = window;
    s.scale = scale;
    s.align = 64;
    s.page_size = page_size;
    s.max_pages = max_pages;
    s.num_pages = num_pages;
    s.page_table = page_table;
    const long long lw = window > 0 ? (long long)window + 63 : (long long)Lmax;
    const int lvis = (int)(lw < Lmax ? lw : Lmax);
    s.splits = num_splits > 0 ? num_splits : auto_splits(Lmax, window);
    int chunk = (lvis + s.splits - 1) / s.splits;
    chunk = (chunk + 63) / 64 * 64;
    s.chunk = chunk;
    s.splits = (lvis + chunk - 1) / chunk;
    return s;
}

size_t decode_ws_bytes(const DecodeShape &s)
{
    if (s.splits <= 1) return 0;
    return (size_t)s.B * s.Hq * s.splits * (s.D + 2) * sizeof(float);
}

}  // namespace

unsigned *device_status_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    return g_dev[dev].status_ptr;
}

long long wait_timeout_ns() { return g_timeout_ns.load(); }

bool encode_tensor_map_4d(void *map, void *gaddr, int elem_bytes, const uint64_t dims[4],
                          const uint64_t strides_bytes[3], const uint32_t box[4], bool swizzle128)
{
    return encode_tensor_map_4d_sw(map, gaddr, elem_bytes, dims, strides_bytes, box, swizzle128 ? 128 : 0);
}

bool encode_tensor_map_4d_sw(void *map, void *gaddr, int elem_bytes, const uint64_t dims[4],
                             const uint64_t strides_bytes[3], const uint32_t box[4], int swizzle_bytes)
{
    std::call_once(g_encode_once, []() {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        else
            cudaGetLastError();
    });
    if (!g_encode || (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4)) return false;
    if (swizzle_bytes != 0 && swizzle_bytes != 64 && swizzle_bytes != 128) return false;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt = elem_bytes == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const CUresult r = g_encode(static_cast<CUtensorMap *>(map), dt, 4, gaddr,
                                reinterpret_cast<const cuuint64_t *>(dims),
                                reinterpret_cast<const cuuint64_t *>(strides_bytes),
                                reinterpret_cast<const cuuint32_t *>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace attn_sink

using namespace attn_sink;

extern "C" {

int attn_sink_version(void) { return 100; }

int attn_sink_last_cuda_error(void) { return g_last_cuda_error; }

const char *attn_sink_strerror(int status)
{
    switch (status) {
    case ATTN_SINK_OK: return "ok";
    case ATTN_SINK_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_SINK_ERR_UNSUPPORTED: return "unsupported configuration (head dim must be 64; dtype f32 or bf16)";
    case ATTN_SINK_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case ATTN_SINK_ERR_ARCH: return "device is not sm_100 (B200); this library only runs on sm_100a";
    case ATTN_SINK_ERR_WORKSPACE: return "workspace missing or too small";
    case ATTN_SINK_ERR_CUDA: return "CUDA call or kernel launch failed";
    case ATTN_SINK_ERR_TIMEOUT: return "a bounded device-side wait expired";
    case ATTN_SINK_ERR_NO_DEVICE: return "no CUDA device visible";
    case ATTN_SINK_ERR_SCRATCH_LIMIT:
        return "problem needs more scratch than the library's built-in no-allocation buffer "
               "(ATTN_SINK_NOALLOC_SCRATCH_BYTES); use fewer splits or attn_sink_decode with a workspace";
    default: return "unknown status";
    }
}

long long attn_sink_set_wait_timeout_ns(long long ns)
{
    return g_timeout_ns.exchange(ns > 0 ? ns : kDefaultTimeoutNs);
}

int attn_sink_fwd(const void *q, const void *k, const void *v, const float *sinks, void *out, float *lse, int B,
                  int Lq, int Lk, int Hq, int Hkv, int D, int window, float scale, int dtype, void *stream)
{
    if (!q || !k || !v || !sinks || !out || !lse) return ATTN_SINK_ERR_INVALID_ARG;
    int rc = check_common(B, Lq, Lk, Hq, Hkv, D, dtype);
    if (rc != ATTN_SINK_OK) return rc;
    // the tensor-core forwards scale the row maximum of the raw scores, which
    // is the maximum of the scaled scores only for a positive scale
    if (dtype == ATTN_SINK_DTYPE_BF16 && !(scale > 0.f && scale < INFINITY)) return ATTN_SINK_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
        !aligned16(sinks))
        return ATTN_SINK_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    AttnShape s{B, Lq, Lk, Hq, Hkv, D, window, scale};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == ATTN_SINK_DTYPE_F32)
        return launch_status(launch_fwd_simt<float>(static_cast<const float *>(q), static_cast<const float *>(k),
                                                    static_cast<const float *>(v), sinks,
                                                    static_cast<float *>(out), lse, s, st));
    if (!fwd_tc_supported(s)) return ATTN_SINK_ERR_UNSUPPORTED;
    return launch_status(launch_fwd_tc(q, k, v, sinks, out, lse, s, st));
}

size_t attn_sink_fwd_host_workspace_size(int B, int Lq, int Lk, int Hq, int Hkv, int D)
{
    if (check_common(B, Lq, Lk, Hq, Hkv, D, ATTN_SINK_DTYPE_BF16) != ATTN_SINK_OK) return 0;
    return fwd_host_workspace_bytes(AttnShape{B, Lq, Lk, Hq, Hkv, D, 0, 1.f});
}

int attn_sink_fwd_host(const void *q_host, const void *k_host, const void *v_host, const float *sinks_host,
                       void *out_host, float *lse_host, int B, int Lq, int Lk, int Hq, int Hkv, int D, int window,
                       float scale, int n_chunks, void *workspace, size_t ws_bytes, void *stream)
{
    if (!q_host || !k_host || !v_host || !sinks_host || !out_host || !lse_host) return ATTN_SINK_ERR_INVALID_ARG;
    if (n_chunks < 1 || n_chunks > kFwdHostMaxChunks) return ATTN_SINK_ERR_INVALID_ARG;
    int rc = check_common(B, Lq, Lk, Hq, Hkv, D, ATTN_SINK_DTYPE_BF16);
    if (rc != ATTN_SINK_OK) return rc;
    if (!(scale > 0.f && scale < INFINITY) || Lq > Lk) return ATTN_SINK_ERR_UNSUPPORTED;
    const AttnShape s{B, Lq, Lk, Hq, Hkv, D, window, scale};
    if (!fwd_tc_supported(s)) return ATTN_SINK_ERR_UNSUPPORTED;
    if (!workspace || ws_bytes < fwd_host_workspace_bytes(s)) return ATTN_SINK_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_SINK_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    return launch_status(run_fwd_host(q_host, k_host, v_host, sinks_host, out_host, lse_host, s, n_chunks, workspace,
                                      static_cast<cudaStream_t>(stream)));
}

size_t attn_sink_fwd_fp8_workspace_size(int B, int Lk, int Hkv, int D)
{
    if (B <= 0 || Lk <= 0 || Hkv <= 0 || D <= 0) return 0;
    AttnShape s{B, 1, Lk, Hkv, Hkv, D, 0, 1.f};
    return fwd_fp8_workspace_bytes(s);
}

int attn_sink_fwd_fp8(const void *q, const void *k, const void *v, const float *q_scale, const float *k_scale,
                      const float *v_scale, const float *sinks, void *out, float *lse, int B, int Lq, int Lk, int Hq,
                      int Hkv, int D, int window, float scale, void *workspace, size_t ws_bytes, void *stream)
{
    if (!q || !k || !v || !q_scale || !k_scale || !v_scale || !sinks || !out || !lse) return ATTN_SINK_ERR_INVALID_ARG;
    int rc = check_common(B, Lq, Lk, Hq, Hkv, D, ATTN_SINK_DTYPE_BF16);
    if (rc != ATTN_SINK_OK) return rc;
    if (!(scale > 0.f && scale < INFINITY)) return ATTN_SINK_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_scale) || !aligned16(k_scale) ||
        !aligned16(v_scale) || !aligned16(out) || !aligned16(lse) || !aligned16(sinks))
        return ATTN_SINK_ERR_MISALIGNED;
    AttnShape s{B, Lq, Lk, Hq, Hkv, D, window, scale};
    if (!workspace || ws_bytes < fwd_fp8_workspace_bytes(s)) return ATTN_SINK_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_SINK_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    if (!fwd_tc_supported(s)) return ATTN_SINK_ERR_UNSUPPORTED;
    return launch_status(launch_fwd_tc_fp8(q, k, v, q_scale, k_scale, v_scale, sinks, out, lse, workspace, s,
                                           static_cast<cudaStream_t>(stream)));
}

int attn_sink_fwd_varlen(const void *q, const void *k, const void *v, const float *sinks, void *out, float *lse,
                         const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int max_seqlen_q, int total_q,
                         int total_k, int Hq, int Hkv, int D, int window, float scale, void *stream)
{
    if (!q || !k || !v || !sinks || !out || !lse || !cu_seqlens_q || !cu_seqlens_k) return ATTN_SINK_ERR_INVALID_ARG;
    int rc = check_common(B, max_seqlen_q, 1, Hq, Hkv, D, ATTN_SINK_DTYPE_BF16);
    if (rc != ATTN_SINK_OK) return rc;
    if (total_q <= 0 || total_k <= 0) return ATTN_SINK_ERR_INVALID_ARG;
    if (!(scale > 0.f && scale < INFINITY)) return ATTN_SINK_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) || !aligned16(sinks) ||
        !aligned16(cu_seqlens_q) || !aligned16(cu_seqlens_k))
        return ATTN_SINK_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    AttnShape s{B, max_seqlen_q, max_seqlen_q, Hq, Hkv, D, window, scale};
    s.cu_q = cu_seqlens_q;
    s.cu_k = cu_seqlens_k;
    s.total_q = total_q;
    s.total_k = total_k;
    if (!fwd_tc_supported(s)) return ATTN_SINK_ERR_UNSUPPORTED;
    return launch_status(launch_fwd_tc(q, k, v, sinks, out, lse, s, static_cast<cudaStream_t>(stream)));
}

int attn_sink_qkv_prologue(const void *qkv, const float *bias, const int *positions, const int *kv_rows, void *q_out,
                           void *k_out, void *v_out, int T, int Hq, int Hkv, int D, int kv_rows_total,
                           float rope_theta, float rope_factor, int rope_original_max_pos, float beta_fast,
                           float beta_slow, int interleaved, void *stream)
{
    if (!qkv || !positions || !q_out || !k_out || !v_out) return ATTN_SINK_ERR_INVALID_ARG;
    if (T <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || kv_rows_total <= 0 || Hq % Hkv != 0)
        return ATTN_SINK_ERR_INVALID_ARG;
    if (D != 64) return ATTN_SINK_ERR_UNSUPPORTED;
    if (!kv_rows && kv_rows_total < T) return ATTN_SINK_ERR_INVALID_ARG;
    if (!(rope_theta > 1.f && rope_theta < INFINITY) || !(rope_factor > 0.f && rope_factor < INFINITY))
        return ATTN_SINK_ERR_INVALID_ARG;
    if (rope_factor > 1.f && (rope_original_max_pos <= 0 || !(beta_fast > beta_slow) || !(beta_slow > 0.f)))
        return ATTN_SINK_ERR_INVALID_ARG;
    if (interleaved != 0 && interleaved != 1) return ATTN_SINK_ERR_INVALID_ARG;
    if (!aligned16(qkv) || !aligned16(positions) || !aligned16(q_out) || !aligned16(k_out) || !aligned16(v_out) ||
        (bias && !aligned16(bias)) || (kv_rows && !aligned16(kv_rows)))
        return ATTN_SINK_ERR_MISALIGNED;
    int rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    const RopeParams r{rope_theta, rope_factor, (double)rope_original_max_pos, beta_fast, beta_slow, interleaved};
    return launch_status(launch_qkv_prologue(qkv, bias, positions, kv_rows, q_out, k_out, v_out, T, Hq, Hkv,
                                             kv_rows_total, r, static_cast<cudaStream_t>(stream)));
}

size_t attn_sink_decode_workspace_size(int B, int Hq, int D, int Lmax, int window, int num_splits)
{
    if (B <= 0 || Hq <= 0 || D <= 0 || Lmax <= 0 || num_splits < 0 || num_splits > 32) return 0;
    return decode_ws_bytes(decode_shape(B, Lmax, Hq, 1, D, window, 1.f, num_splits));
}

int attn_sink_decode(const void *q, const void *k_cache, const void *v_cache, const int *seqlens,
                     const float *sinks, void *out, float *lse, int B, int Lmax, int Hq, int Hkv, int D,
                     int window, float scale, int num_splits, void *workspace, size_t ws_bytes, int dtype,
                     void *stream)
{
    if (!q || !k_cache || !v_cache || !seqlens || !sinks || !out || !lse) return ATTN_SINK_ERR_INVALID_ARG;
    if (num_splits < 0 || num_splits > 32) return ATTN_SINK_ERR_INVALID_ARG;
    int rc = check_common(B, 1, Lmax, Hq, Hkv, D, dtype);
    if (rc != ATTN_SINK_OK) return rc;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(lse) ||
        !aligned16(sinks) || !aligned16(seqlens))
        return ATTN_SINK_ERR_MISALIGNED;
    const DecodeShape s = decode_shape(B, Lmax, Hq, Hkv, D, window, scale, num_splits);
    const size_t need = decode_ws_bytes(s);
    if (need > 0 && (!workspace || ws_bytes < need)) return ATTN_SINK_ERR_WORKSPACE;
    if (need > 0 && !aligned16(workspace)) return ATTN_SINK_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *ws_o = static_cast<float *>(workspace);
    float *ws_ml = need > 0 ? ws_o + (size_t)s.B * s.Hq * s.splits * s.D : nullptr;
    cudaError_t e;
    if (dtype == ATTN_SINK_DTYPE_F32) {
        e = launch_decode_simt<float>(static_cast<const float *>(q), static_cast<const float *>(k_cache),
                                      static_cast<const float *>(v_cache), seqlens, sinks,
                                      static_cast<float *>(out), lse, s, ws_o, ws_ml, st);
        if (e == cudaSuccess && s.splits > 1)
            e = launch_decode_combine<float>(seqlens, sinks, static_cast<float *>(out), lse, s, ws_o, ws_ml, st);
    } else {
        if (decode_bf16_supported(s))
            e = launch_decode_bf16(q, k_cache, v_cache, seqlens, sinks, out, lse, s, ws_o, ws_ml, st);
        else
            e = launch_decode_simt<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(q),
                                                  static_cast<const __nv_bfloat16 *>(k_cache),
                                                  static_cast<const __nv_bfloat16 *>(v_cache), seqlens, sinks,
                                                  static_cast<__nv_bfloat16 *>(out), lse, s, ws_o, ws_ml, st);
        if (e == cudaSuccess && s.splits > 1)
            e = launch_decode_combine<__nv_bfloat16>(seqlens, sinks, static_cast<__nv_bfloat16 *>(out), lse, s,
                                                     ws_o, ws_ml, st);
    }
    return launch_status(e);
}

int attn_sink_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const float *k_scale,
                         const float *v_scale, const int *seqlens, const float *sinks, void *out, float *lse, int B,
                         int Lmax, int Hq, int Hkv, int D, int window, float scale, int num_splits, void *workspace,
                         size_t ws_bytes, void *stream)
{
    if (!q || !k_cache || !v_cache || !k_scale || !v_scale || !seqlens || !sinks || !out || !lse)
        return ATTN_SINK_ERR_INVALID_ARG;
    if (num_splits < 0 || num_splits > 32) return ATTN_SINK_ERR_INVALID_ARG;
    int rc = check_common(B, 1, Lmax, Hq, Hkv, D, ATTN_SINK_DTYPE_BF16);
    if (rc != ATTN_SINK_OK) return rc;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_scale) || !aligned16(v_scale) ||
        !aligned16(out) || !aligned16(lse) || !aligned16(sinks) || !aligned16(seqlens))
        return ATTN_SINK_ERR_MISALIGNED;
    DecodeShape s = decode_shape(B, Lmax, Hq, Hkv, D, window, scale, num_splits);
    // the e4m3 kernel's tiles are 128 keys: chunks of whole tiles (never more
    // splits than the bf16 rule, so the same workspace size suffices)
    const int lvis = window > 0 ? (window < Lmax ? window : Lmax) : Lmax;
    s.chunk = (s.chunk + 127) / 128 * 128;
    s.splits = (lvis + s.chunk - 1) / s.chunk;
    if (!decode_bf16_supported(s)) return ATTN_SINK_ERR_UNSUPPORTED;
    const size_t need = decode_ws_bytes(s);
    if (need > 0 && (!workspace || ws_bytes < need)) return ATTN_SINK_ERR_WORKSPACE;
    if (need > 0 && !aligned16(workspace)) return ATTN_SINK_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *ws_o = static_cast<float *>(workspace);
    float *ws_ml = need > 0 ? ws_o + (size_t)s.B * s.Hq * s.splits * s.D : nullptr;
    cudaError_t e = launch_decode_bf16(q, k_cache, v_cache, seqlens, sinks, out, lse, s, ws_o, ws_ml, st, k_scale,
                                       v_scale);
    if (e == cudaSuccess && s.splits > 1)
        e = launch_decode_combine<__nv_bfloat16>(seqlens, sinks, static_cast<__nv_bfloat16 *>(out), lse, s, ws_o,
                                                 ws_ml, st);
    return launch_status(e);
}

size_t attn_sink_decode_paged_workspace_size(int B, int Hq, int D, int max_pages_per_seq, int page_size, int window,
                                             int num_splits)
{
    if (B <= 0 || Hq <= 0 || D <= 0 || num_splits < 0 || num_splits > 32) return 0;
    if (!paged_sizes_ok(page_size, max_pages_per_seq, 1)) return 0;
    return decode_ws_bytes(
        decode_shape_paged(B, max_pages_per_seq, page_size, 1, nullptr, Hq, 1, D, window, 1.f, num_splits));
}

int attn_sink_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int *page_table,
                           const int *seqlens, const float *sinks, void *out, float *lse, int B,
                           int max_pages_per_seq, int page_size, int num_pages, int Hq, int Hkv, int D, int window,
                           float scale, int num_splits, void *workspace, size_t ws_bytes, int dtype, void *stream)
{
    if (!q || !k_pages || !v_pages || !page_table || !seqlens || !sinks || !out || !lse)
        return ATTN_SINK_ERR_INVALID_ARG;
    if (num_splits < 0 || num_splits > 32) return ATTN_SINK_ERR_INVALID_ARG;
    if (!paged_sizes_ok(page_size, max_pages_per_seq, num_pages)) return ATTN_SINK_ERR_INVALID_ARG;
    int rc = check_common(B, 1, max_pages_per_seq * page_size, Hq, Hkv, D, dtype);
    if (rc != ATTN_SINK_OK) return rc;
    if (dtype != ATTN_SINK_DTYPE_BF16) return ATTN_SINK_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(page_table) || !aligned16(out) ||
        !aligned16(lse) || !aligned16(sinks) || !aligned16(seqlens))
        return ATTN_SINK_ERR_MISALIGNED;
    const DecodeShape s = decode_shape_paged(B, max_pages_per_seq, page_size, num_pages, page_table, Hq, Hkv, D,
                                             window, scale, num_splits);
    if (!decode_bf16_supported(s)) return ATTN_SINK_ERR_UNSUPPORTED;
    const size_t need = decode_ws_bytes(s);
    if (need > 0 && (!workspace || ws_bytes < need)) return ATTN_SINK_ERR_WORKSPACE;
    if (need > 0 && !aligned16(workspace)) return ATTN_SINK_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *ws_o = static_cast<float *>(workspace);
    float *ws_ml = need > 0 ? ws_o + (size_t)s.B * s.Hq * s.splits * s.D : nullptr;
    cudaError_t e = launch_decode_bf16(q, k_pages, v_pages, seqlens, sinks, out, lse, s, ws_o, ws_ml, st);
    if (e == cudaSuccess && s.splits > 1)
        e = launch_decode_combine<__nv_bfloat16>(seqlens, sinks, static_cast<__nv_bfloat16 *>(out), lse, s, ws_o,
                                                 ws_ml, st);
    return launch_status(e);
}

namespace {
// bf16 backward workspace: [D_i][dsink terms] (as the exact path) + fp32 dQ accumulator
size_t bwd_ws_bytes(const AttnShape &s, int dtype)
{
    const size_t base = (bwd_simt_workspace_bytes(s) + 255) / 256 * 256;
    return dtype == ATTN_SINK_DTYPE_F32 ? bwd_simt_workspace_bytes(s) : base + bwd_tc_dq_acc_bytes(s);
}
}  // namespace

size_t attn_sink_bwd_workspace_size(int B, int Lq, int Lk, int Hq, int Hkv, int D, int dtype)
{
    if (check_common(B, Lq, Lk, Hq, Hkv, D, dtype) != ATTN_SINK_OK) return 0;
    AttnShape s{B, Lq, Lk, Hq, Hkv, D, 0, 1.f};
    return bwd_ws_bytes(s, dtype);
}

int attn_sink_bwd(const void *q, const void *k, const void *v, const float *sinks, const void *out,
                  const void *dout, const float *lse, void *dq, void *dk, void *dv, float *dsinks, int B, int Lq,
                  int Lk, int Hq, int Hkv, int D, int window, float scale, void *workspace, size_t ws_bytes,
                  int dtype, void *stream)
{
    if (!q || !k || !v || !sinks || !out || !dout || !lse || !dq || !dk || !dv || !dsinks)
        return ATTN_SINK_ERR_INVALID_ARG;
    int rc = check_common(B, Lq, Lk, Hq, Hkv, D, dtype);
    if (rc != ATTN_SINK_OK) return rc;
    const void *ptrs[] = {q, k, v, sinks, out, dout, lse, dq, dk, dv, dsinks};
    for (const void *p : ptrs)
        if (!aligned16(p)) return ATTN_SINK_ERR_MISALIGNED;
    AttnShape s{B, Lq, Lk, Hq, Hkv, D, window, scale};
    const size_t need = bwd_ws_bytes(s, dtype);
    if (!workspace || ws_bytes < need) return ATTN_SINK_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_SINK_ERR_MISALIGNED;
    rc = ensure_device();
    if (rc != ATTN_SINK_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == ATTN_SINK_DTYPE_F32)
        return launch_status(launch_bwd_simt<float>(
            static_cast<const float *>(q), static_cast<const float *>(k), static_cast<const float *>(v), sinks,
            static_cast<const float *>(out), static_cast<const float *>(dout), lse, static_cast<float *>(dq),
            static_cast<float *>(dk), static_cast<float *>(dv), dsinks, s, workspace, st));
    using bf = __nv_bfloat16;
    if (!bwd_tc_supported(s)) return ATTN_SINK_ERR_UNSUPPORTED;
    const size_t rows = (size_t)B * Hq * Lq;
    float *Drow = static_cast<float *>(workspace);
    float *terms = Drow + rows;
    float *dq_acc = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                              (bwd_simt_workspace_bytes(s) + 255) / 256 * 256);
    // the row pre-pass also clears the dQ accumulator the main pass adds into
    cudaError_t e = launch_bwd_rows<bf>(static_cast<const bf *>(out), static_cast<const bf *>(dout), lse, sinks, Drow,
                                        terms, dq_acc, s, st);
    if (e == cudaSuccess) e = launch_bwd_tc(q, k, v, dout, lse, Drow, terms, dsinks, dq_acc, dq, dk, dv, s, st);
    return launch_status(e);
}

int attn_sink_get_device_status(void *stream)
{
    int dev = 0;
    int rc = current_device(&dev);
    if (rc != ATTN_SINK_OK) return rc;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_SINK_ERR_CUDA;
    }
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_SINK_ERR_CUDA;
    }
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_SINK_ERR_CUDA;
        }
    }
    return (v & STATUS_TIMEOUT) ? ATTN_SINK_ERR_TIMEOUT : ATTN_SINK_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any allocation: the split partials live in a file-scope
// device array.  In host code `g_noalloc_scratch` names a host-side shadow,
// not device memory, so the kernels get the device address looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_SINK_NOALLOC_SCRATCH_BYTES];

namespace {

struct NoAllocScratch {
    std::once_flag once;
    int status = ATTN_SINK_ERR_CUDA;
    void *ptr = nullptr;
};
NoAllocScratch g_noalloc[kMaxDevices];

// Once per device, with that device current: device address of the array.
int noalloc_scratch(void **ptr)
{
    int dev = 0;
    int rc = current_device(&dev);
    if (rc != ATTN_SINK_OK) return rc;
    NoAllocScratch &s = g_noalloc[dev];
    std::call_once(s.once, [&s]() {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            s.status = ATTN_SINK_ERR_CUDA;
            return;
        }
        s.ptr = p;
        s.status = ATTN_SINK_OK;
    });
    *ptr = s.ptr;
    return s.status;
}

}  // namespace

extern "C" int attn_sink_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                        const int *seqlens, const float *sinks, void *out, float *lse, int B,
                                        int Lmax, int Hq, int Hkv, int D, int window, float scale,
                                        int num_splits, int dtype, void *stream)
{
    if (num_splits < 0 || num_splits > 32) return ATTN_SINK_ERR_INVALID_ARG;
    const int rc0 = check_common(B, 1, Lmax, Hq, Hkv, D, dtype);
    if (rc0 != ATTN_SINK_OK) return rc0;
    const size_t need = decode_ws_bytes(decode_shape(B, Lmax, Hq, Hkv, D, window, scale, num_splits));
    if (need > ATTN_SINK_NOALLOC_SCRATCH_BYTES) return ATTN_SINK_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if (need > 0) {
        int rc = ensure_device();
        if (rc != ATTN_SINK_OK) return rc;
        rc = noalloc_scratch(&scratch);
        if (rc != ATTN_SINK_OK) return rc;
    }
    return attn_sink_decode(q, k_cache, v_cache, seqlens, sinks, out, lse, B, Lmax, Hq, Hkv, D, window, scale,
                            num_splits, scratch, need > 0 ? (size_t)ATTN_SINK_NOALLOC_SCRATCH_BYTES : 0, dtype,
                            stream);
}
