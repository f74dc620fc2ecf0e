"""attn_sink_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (their memory belongs to a host framework or server
allocator, or their decode loop cannot afford a cudaMalloc).  It must give
the same result as attn_sink_decode with a caller workspace, call after call,
although every call reuses the library's one built-in scratch array.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test; it also passes alone.
"""
import ctypes
import math

import pytest
import torch

import gqa_softmax_attention_attn_b200 as attn
from _harness import assert_close_bf16, assert_lse
from gqa_softmax_attention_attn_b200.inputs import decode_inputs

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = -9


def _reference(d, window, splits):
    B, Hq, D = d["q"].shape
    Lmax = d["k_cache"].shape[1]
    out = torch.empty_like(d["q"])
    lse = torch.empty(B, Hq, device="cuda", dtype=torch.float32)
    nbytes = attn.attn_sink_decode_workspace_size(B, Hq, D, Lmax, window, splits)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    attn.attn_sink_decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"], out, lse, window,
                          1.0 / math.sqrt(D), splits, ws)
    return out, lse


def _noalloc_via_abi(d, window, splits):
    """Calls the C entry point directly through ctypes (no Python wrapper)."""
    lib = attn.load()
    B, Hq, D = d["q"].shape
    Lmax, Hkv = d["k_cache"].shape[1], d["k_cache"].shape[2]
    out = torch.full_like(d["q"], float("nan"))
    lse = torch.full((B, Hq), float("nan"), device="cuda", dtype=torch.float32)
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.attn_sink_decode_noalloc(
        ctypes.c_void_p(d["q"].data_ptr()), ctypes.c_void_p(d["k_cache"].data_ptr()),
        ctypes.c_void_p(d["v_cache"].data_ptr()), ctypes.c_void_p(d["seqlens"].data_ptr()),
        ctypes.c_void_p(d["sinks"].data_ptr()), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        B, Lmax, Hq, Hkv, D, window, ctypes.c_float(1.0 / math.sqrt(D)), splits, attn.DTYPE_BF16,
        ctypes.c_void_p(stream))
    assert rc == 0, attn.strerror(rc)
    return out, lse


@pytest.mark.parametrize("window,splits", [(0, 0), (0, 8), (128, 0), (0, 32)])
def test_noalloc_decode_matches_workspace_decode_two_calls_in_a_row(window, splits):
    torch.manual_seed(0)
    d = decode_inputs(16, 8192, 64, 8, 64, 100, 8192, torch.bfloat16, 0.5, 1.0, seed=41 + splits)
    d = {k: v.cuda() for k, v in d.items()}
    ref_out, ref_lse = _reference(d, window, splits)
    for call in range(2):
        out, lse = _noalloc_via_abi(d, window, splits)
        torch.cuda.synchronize()
        assert_close_bf16(out, ref_out, f"noalloc call {call} w={window} s={splits}")
        assert_lse(lse, ref_lse, f"noalloc call {call} w={window} s={splits}")
    assert attn.attn_sink_get_device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    """B=512, Hq=64, 32 splits needs 512*64*32*66*4 bytes > 32 MiB: rejected on the host."""
    lib = attn.load()
    need = attn.attn_sink_decode_workspace_size(512, 64, 64, 32768, 0, 32)
    assert need > attn._native.NOALLOC_SCRATCH_BYTES
    fake = [ctypes.c_void_p(0x7f0000000000 + 0x1000 * i) for i in range(7)]
    rc = lib.attn_sink_decode_noalloc(*fake, 512, 32768, 64, 8, 64, 0, ctypes.c_float(0.125), 32,
                                      attn.DTYPE_BF16, None)
    assert rc == SCRATCH_LIMIT
    assert "scratch" in attn.strerror(rc)
