"""ctypes binding of libattn_sink.so -- argument marshalling only.

Every function here has the name of the C entry point it calls
(include/attn_sink.h) and does nothing but check tensor shapes/devices,
take data pointers and raise on a non-zero status.  All arithmetic runs in the
library's CUDA kernels; there is no CPU or library fallback.  If the shared
library is missing the first call raises ``AttnSinkLibraryMissing``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libattn_sink.so")

DTYPE_F32 = 0
DTYPE_BF16 = 1

_lock = threading.Lock()
_lib = None


class AttnSinkLibraryMissing(RuntimeError):
    pass


class AttnSinkError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: status {status} ({strerror(status)})"
        if status == -6:
            code = attn_sink_last_cuda_error()
            try:
                import ctypes.util

                rt = torch.cuda.cudart()
                name = rt.cudaGetErrorString(code) if hasattr(rt, "cudaGetErrorString") else ""
            except Exception:
                name = ""
            msg += f"; CUDA error {code} {name}"
        super().__init__(msg)


def load():
    """Loads the in-tree libattn_sink.so (built by gqa_softmax_attention_attn_b200.build)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise AttnSinkLibraryMissing(
                f"{LIB_PATH} not found: build it with `python -m gqa_softmax_attention_attn_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, F, Z, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_longlong
        lib.attn_sink_fwd.argtypes = [P] * 6 + [I] * 7 + [F, I, P]
        lib.attn_sink_fwd.restype = I
        lib.attn_sink_qkv_prologue.argtypes = [P] * 7 + [I] * 5 + [F, F, I, F, F, I, P]
        lib.attn_sink_qkv_prologue.restype = I
        lib.attn_sink_fwd_varlen.argtypes = [P] * 8 + [I] * 8 + [F, P]
        lib.attn_sink_fwd_varlen.restype = I
        lib.attn_sink_decode.argtypes = [P] * 7 + [I] * 6 + [F, I, P, Z, I, P]
        lib.attn_sink_decode.restype = I
        lib.attn_sink_decode_noalloc.argtypes = [P] * 7 + [I] * 6 + [F, I, I, P]
        lib.attn_sink_decode_noalloc.restype = I
        lib.attn_sink_decode_workspace_size.argtypes = [I] * 6
        lib.attn_sink_decode_workspace_size.restype = Z
        lib.attn_sink_decode_fp8.argtypes = [P] * 9 + [I] * 6 + [F, I, P, Z, P]
        lib.attn_sink_decode_fp8.restype = I
        lib.attn_sink_fwd_fp8.argtypes = [P] * 9 + [I] * 7 + [F, P, Z, P]
        lib.attn_sink_fwd_fp8.restype = I
        lib.attn_sink_fwd_fp8_workspace_size.argtypes = [I] * 4
        lib.attn_sink_fwd_fp8_workspace_size.restype = Z
        lib.attn_sink_fwd_host.argtypes = [P] * 6 + [I] * 7 + [F, I, P, Z, P]
        lib.attn_sink_fwd_host.restype = I
        lib.attn_sink_fwd_host_workspace_size.argtypes = [I] * 6
        lib.attn_sink_fwd_host_workspace_size.restype = Z
        lib.attn_sink_decode_paged.argtypes = [P] * 8 + [I] * 8 + [F, I, P, Z, I, P]
        lib.attn_sink_decode_paged.restype = I
        lib.attn_sink_decode_paged_workspace_size.argtypes = [I] * 7
        lib.attn_sink_decode_paged_workspace_size.restype = Z
        lib.attn_sink_bwd.argtypes = [P] * 11 + [I] * 7 + [F, P, Z, I, P]
        lib.attn_sink_bwd.restype = I
        lib.attn_sink_bwd_workspace_size.argtypes = [I] * 7
        lib.attn_sink_bwd_workspace_size.restype = Z
        lib.attn_sink_get_device_status.argtypes = [P]
        lib.attn_sink_get_device_status.restype = I
        lib.attn_sink_set_wait_timeout_ns.argtypes = [LL]
        lib.attn_sink_set_wait_timeout_ns.restype = LL
        lib.attn_sink_strerror.argtypes = [I]
        lib.attn_sink_strerror.restype = ctypes.c_char_p
        lib.attn_sink_version.argtypes = []
        lib.attn_sink_version.restype = I
        lib.attn_sink_last_cuda_error.argtypes = []
        lib.attn_sink_last_cuda_error.restype = I
        _lib = lib
        return lib


def strerror(status: int) -> str:
    return load().attn_sink_strerror(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DTYPE_F32
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _host(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise AttnSinkError(rc, where)


def attn_sink_fwd(q, k, v, sinks, out, lse, window: int, scale: float, stream=None):
    """q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D], sinks [Hq] fp32 -> writes out [B,Lq,Hq,D], lse [B,Hq,Lq] fp32."""
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    dt = q.dtype
    rc = load().attn_sink_fwd(_dev(q, "q"), _dev(k, "k", dt), _dev(v, "v", dt), _dev(sinks, "sinks", torch.float32),
                              _dev(out, "out", dt), _dev(lse, "lse", torch.float32), B, Lq, Lk, Hq, Hkv, D,
                              int(window), float(scale), _dtype_code(q), _stream(stream))
    _check(rc, "attn_sink_fwd")


def attn_sink_fwd_host_workspace_size(B: int, Lq: int, Lk: int, Hq: int, Hkv: int, D: int) -> int:
    return int(load().attn_sink_fwd_host_workspace_size(B, Lq, Lk, Hq, Hkv, D))


def attn_sink_fwd_host(q, k, v, sinks, out, lse, window: int, scale: float, workspace, n_chunks: int = 8,
                       stream=None):
    """The bf16 prefill forward on HOST tensors (pin them for the copies to overlap): q [B,Lq,Hq,D],
    k/v [B,Lk,Hkv,D] bf16, sinks [Hq] fp32 -> writes out [B,Lq,Hq,D] bf16, lse [B,Hq,Lq] fp32 in host
    memory; workspace: a CUDA tensor of attn_sink_fwd_host_workspace_size bytes.  Asynchronous on
    `stream`: synchronise it before reading out or lse."""
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    bf = torch.bfloat16
    rc = load().attn_sink_fwd_host(_host(q, "q", bf), _host(k, "k", bf), _host(v, "v", bf),
                                   _host(sinks, "sinks", torch.float32), _host(out, "out", bf),
                                   _host(lse, "lse", torch.float32), B, Lq, Lk, Hq, Hkv, D, int(window), float(scale),
                                   int(n_chunks), _dev(workspace, "workspace"),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "attn_sink_fwd_host")


def attn_sink_qkv_prologue(qkv, bias, positions, q_out, k_out, v_out, rope_theta: float, rope_factor: float = 1.0,
                           rope_original_max_pos: int = 0, beta_fast: float = 32.0, beta_slow: float = 1.0,
                           interleaved: bool = False, kv_rows=None, stream=None):
    """qkv [T,(Hq+2Hkv)*D] bf16, bias [(Hq+2Hkv)*D] fp32 or None, positions [T] int32 -> writes
    q_out [T,Hq,D], k_out/v_out [rows,Hkv,D] (row kv_rows[t], or t) with bias and YaRN rotary embedding."""
    T, Hq, D = q_out.shape
    rows, Hkv = k_out.shape[0], k_out.shape[1]
    if qkv.shape != (T, (Hq + 2 * Hkv) * D):
        raise ValueError(f"qkv must be [{T}, {(Hq + 2 * Hkv) * D}]")
    rc = load().attn_sink_qkv_prologue(_dev(qkv, "qkv", torch.bfloat16),
                                       _dev(bias, "bias", torch.float32) if bias is not None else None,
                                       _dev(positions, "positions", torch.int32),
                                       _dev(kv_rows, "kv_rows", torch.int32) if kv_rows is not None else None,
                                       _dev(q_out, "q_out", torch.bfloat16), _dev(k_out, "k_out", torch.bfloat16),
                                       _dev(v_out, "v_out", torch.bfloat16), T, Hq, Hkv, D, rows, float(rope_theta),
                                       float(rope_factor), int(rope_original_max_pos), float(beta_fast),
                                       float(beta_slow), int(bool(interleaved)), _stream(stream))
    _check(rc, "attn_sink_qkv_prologue")


def attn_sink_fwd_varlen(q, k, v, sinks, out, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, window: int,
                         scale: float, stream=None):
    """Packed ragged sequences: q [total_q,Hq,D], k/v [total_k,Hkv,D] bf16, cu_seqlens_q/k [B+1] int32
    -> writes out [total_q,Hq,D], lse [Hq,total_q]."""
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.shape[0] - 1
    if cu_seqlens_k.shape[0] != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold B + 1 offsets")
    rc = load().attn_sink_fwd_varlen(_dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16),
                                     _dev(v, "v", torch.bfloat16), _dev(sinks, "sinks", torch.float32),
                                     _dev(out, "out", torch.bfloat16), _dev(lse, "lse", torch.float32),
                                     _dev(cu_seqlens_q, "cu_seqlens_q", torch.int32),
                                     _dev(cu_seqlens_k, "cu_seqlens_k", torch.int32), B, int(max_seqlen_q), total_q,
                                     total_k, Hq, Hkv, D, int(window), float(scale), _stream(stream))
    _check(rc, "attn_sink_fwd_varlen")


def attn_sink_decode_workspace_size(B: int, Hq: int, D: int, Lmax: int, window: int, num_splits: int) -> int:
    return int(load().attn_sink_decode_workspace_size(B, Hq, D, Lmax, int(window), int(num_splits)))


def attn_sink_decode(q, k_cache, v_cache, seqlens, sinks, out, lse, window: int, scale: float,
                     num_splits: int = 0, workspace=None, stream=None):
    """q [B,Hq,D], caches [B,Lmax,Hkv,D], seqlens [B] int32 -> writes out [B,Hq,D], lse [B,Hq]."""
    B, Hq, D = q.shape
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    dt = q.dtype
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = load().attn_sink_decode(_dev(q, "q"), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
                                 _dev(seqlens, "seqlens", torch.int32), _dev(sinks, "sinks", torch.float32),
                                 _dev(out, "out", dt), _dev(lse, "lse", torch.float32), B, Lmax, Hq, Hkv, D,
                                 int(window), float(scale), int(num_splits), ws_ptr, ws_bytes, _dtype_code(q),
                                 _stream(stream))
    _check(rc, "attn_sink_decode")


def attn_sink_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, seqlens, sinks, out, lse, window: int,
                         scale: float, num_splits: int = 0, workspace=None, stream=None):
    """q [B,Hq,D] bf16, caches [B,Lmax,Hkv,D] e4m3 codes (uint8 or float8_e4m3fn), k_scale/v_scale [Hkv]
    fp32, seqlens [B] int32 -> writes out [B,Hq,D] bf16, lse [B,Hq]."""
    B, Hq, D = q.shape
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    for name, c in (("k_cache", k_cache), ("v_cache", v_cache)):
        if c.element_size() != 1:
            raise TypeError(f"{name} must hold one-byte e4m3 codes, got {c.dtype}")
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = load().attn_sink_decode_fp8(_dev(q, "q", torch.bfloat16), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                     _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
                                     _dev(seqlens, "seqlens", torch.int32), _dev(sinks, "sinks", torch.float32),
                                     _dev(out, "out", torch.bfloat16), _dev(lse, "lse", torch.float32), B, Lmax, Hq,
                                     Hkv, D, int(window), float(scale), int(num_splits), ws_ptr, ws_bytes,
                                     _stream(stream))
    _check(rc, "attn_sink_decode_fp8")


def attn_sink_fwd_fp8_workspace_size(B: int, Lk: int, Hkv: int, D: int) -> int:
    return int(load().attn_sink_fwd_fp8_workspace_size(B, Lk, Hkv, D))


def attn_sink_fwd_fp8(q, k, v, q_scale, k_scale, v_scale, sinks, out, lse, window: int, scale: float, workspace,
                      stream=None):
    """q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D] e4m3 codes (uint8 or float8_e4m3fn), q_scale [Hq], k_scale/v_scale
    [Hkv] fp32, workspace of attn_sink_fwd_fp8_workspace_size bytes -> writes out [B,Lq,Hq,D] bf16,
    lse [B,Hq,Lq]."""
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    for name, c in (("q", q), ("k", k), ("v", v)):
        if c.element_size() != 1:
            raise TypeError(f"{name} must hold one-byte e4m3 codes, got {c.dtype}")
    rc = load().attn_sink_fwd_fp8(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(q_scale, "q_scale", torch.float32),
                                  _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
                                  _dev(sinks, "sinks", torch.float32), _dev(out, "out", torch.bfloat16),
                                  _dev(lse, "lse", torch.float32), B, Lq, Lk, Hq, Hkv, D, int(window), float(scale),
                                  _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                  _stream(stream))
    _check(rc, "attn_sink_fwd_fp8")


def attn_sink_decode_paged_workspace_size(B: int, Hq: int, D: int, max_pages_per_seq: int, page_size: int,
                                          window: int, num_splits: int) -> int:
    return int(load().attn_sink_decode_paged_workspace_size(B, Hq, D, max_pages_per_seq, page_size, int(window),
                                                            int(num_splits)))


def attn_sink_decode_paged(q, k_pages, v_pages, page_table, seqlens, sinks, out, lse, window: int, scale: float,
                           num_splits: int = 0, workspace=None, stream=None):
    """q [B,Hq,D], page pools k/v [num_pages,page_size,Hkv,D] bf16, page_table [B,max_pages] int32,
    seqlens [B] int32 -> writes out [B,Hq,D], lse [B,Hq]."""
    B, Hq, D = q.shape
    num_pages, page_size, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    max_pages = page_table.shape[1]
    dt = q.dtype
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = load().attn_sink_decode_paged(_dev(q, "q"), _dev(k_pages, "k_pages", dt), _dev(v_pages, "v_pages", dt),
                                       _dev(page_table, "page_table", torch.int32),
                                       _dev(seqlens, "seqlens", torch.int32), _dev(sinks, "sinks", torch.float32),
                                       _dev(out, "out", dt), _dev(lse, "lse", torch.float32), B, max_pages, page_size,
                                       num_pages, Hq, Hkv, D, int(window), float(scale), int(num_splits), ws_ptr,
                                       ws_bytes, _dtype_code(q), _stream(stream))
    _check(rc, "attn_sink_decode_paged")


NOALLOC_SCRATCH_BYTES = 32 << 20  # ATTN_SINK_NOALLOC_SCRATCH_BYTES


def attn_sink_decode_noalloc(q, k_cache, v_cache, seqlens, sinks, out, lse, window: int, scale: float,
                             num_splits: int = 0, stream=None):
    """attn_sink_decode with the library's built-in scratch instead of a caller workspace
    (for callers that cannot allocate device memory; calls on one device must not overlap)."""
    B, Hq, D = q.shape
    Lmax, Hkv = k_cache.shape[1], k_cache.shape[2]
    dt = q.dtype
    rc = load().attn_sink_decode_noalloc(_dev(q, "q"), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
                                         _dev(seqlens, "seqlens", torch.int32), _dev(sinks, "sinks", torch.float32),
                                         _dev(out, "out", dt), _dev(lse, "lse", torch.float32), B, Lmax, Hq, Hkv, D,
                                         int(window), float(scale), int(num_splits), _dtype_code(q), _stream(stream))
    _check(rc, "attn_sink_decode_noalloc")


def attn_sink_bwd_workspace_size(B: int, Lq: int, Lk: int, Hq: int, Hkv: int, D: int, dtype: int) -> int:
    return int(load().attn_sink_bwd_workspace_size(B, Lq, Lk, Hq, Hkv, D, dtype))


def attn_sink_bwd(q, k, v, sinks, out, dout, lse, dq, dk, dv, dsinks, window: int, scale: float,
                  workspace, stream=None):
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    dt = q.dtype
    rc = load().attn_sink_bwd(_dev(q, "q"), _dev(k, "k", dt), _dev(v, "v", dt), _dev(sinks, "sinks", torch.float32),
                              _dev(out, "out", dt), _dev(dout, "dout", dt), _dev(lse, "lse", torch.float32),
                              _dev(dq, "dq", dt), _dev(dk, "dk", dt), _dev(dv, "dv", dt),
                              _dev(dsinks, "dsinks", torch.float32), B, Lq, Lk, Hq, Hkv, D, int(window),
                              float(scale), _dev(workspace, "workspace"),
                              workspace.numel() * workspace.element_size(), _dtype_code(q), _stream(stream))
    _check(rc, "attn_sink_bwd")


def attn_sink_get_device_status(stream=None) -> int:
    return int(load().attn_sink_get_device_status(_stream(stream)))


def attn_sink_set_wait_timeout_ns(ns: int) -> int:
    return int(load().attn_sink_set_wait_timeout_ns(int(ns)))


def attn_sink_version() -> int:
    return int(load().attn_sink_version())


def attn_sink_last_cuda_error() -> int:
    return int(load().attn_sink_last_cuda_error())
