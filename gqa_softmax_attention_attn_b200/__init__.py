"""Sink-softmax grouped-query attention (gpt-oss style) for NVIDIA B200 (sm_100a).

The kernels live in ``lib/libattn_sink.so`` (C ABI: ``include/attn_sink.h``);
``_native`` is its ctypes binding.  The library is loaded lazily on the first
call, and a call fails loudly when the library is missing: there is no
fallback implementation.
"""
from ._native import (  # noqa: F401
    DTYPE_BF16,
    DTYPE_F32,
    AttnSinkError,
    AttnSinkLibraryMissing,
    attn_sink_bwd,
    attn_sink_bwd_workspace_size,
    attn_sink_decode,
    attn_sink_decode_fp8,
    attn_sink_fwd_fp8,
    attn_sink_fwd_fp8_workspace_size,
    attn_sink_decode_noalloc,
    attn_sink_decode_paged,
    attn_sink_decode_paged_workspace_size,
    attn_sink_decode_workspace_size,
    attn_sink_fwd,
    attn_sink_fwd_host,
    attn_sink_fwd_host_workspace_size,
    attn_sink_fwd_varlen,
    attn_sink_get_device_status,
    attn_sink_qkv_prologue,
    attn_sink_set_wait_timeout_ns,
    attn_sink_version,
    load,
    strerror,
)
