"""Failure detection without a GPU fault: every device-side wait is bounded,
and an expired wait raises a status the host reads, leaving the context usable.

* A self-test kernel waits on an mbarrier that nothing ever arrives on; the
  wait must give up, raise the abort flag and the status bit, and return.
* Through the public API: with the wait limit set to 1 ns, a decode call's
  waits expire; attn_sink_get_device_status reports ATTN_SINK_ERR_TIMEOUT once
  (and clears it), and the next call with the default limit is correct.
"""
import ctypes
import math

import pytest
import torch

import gqa_softmax_attention_attn_b200 as attn
from _harness import assert_close_bf16
from gqa_softmax_attention_attn_b200 import build
from gqa_softmax_attention_attn_b200.inputs import decode_inputs

pytestmark = pytest.mark.gpu
TIMEOUT = -7


def test_bounded_wait_on_a_barrier_nothing_arrives_on():
    lib = ctypes.CDLL(build.SELFTEST_LIB)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    result = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    rc = lib.attn_sink_selftest_timeout(ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(result.data_ptr()),
                                        ctypes.c_longlong(2_000_000), ctypes.c_void_p(0))
    assert rc == 0
    torch.cuda.synchronize()
    assert result.tolist() == [1, 1]
    assert status.item() & 1


def test_expired_waits_are_reported_and_the_context_stays_usable():
    d = decode_inputs(4, 4096, 16, 2, 64, 1000, 4096, torch.bfloat16, 0.5, 1.0, seed=51)
    d = {k: v.cuda() for k, v in d.items()}
    out = torch.empty_like(d["q"])
    lse = torch.empty(4, 16, device="cuda")
    ws = torch.empty(max(16, attn.attn_sink_decode_workspace_size(4, 16, 64, 4096, 0, 8)), dtype=torch.uint8,
                     device="cuda")
    assert attn.attn_sink_get_device_status() == 0
    old = attn.attn_sink_set_wait_timeout_ns(1)
    try:
        attn.attn_sink_decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"], out, lse, 0, 0.125, 8, ws)
        st = attn.attn_sink_get_device_status()
    finally:
        attn.attn_sink_set_wait_timeout_ns(old)
    assert st in (0, TIMEOUT)  # a wait that never had to spin cannot expire
    assert attn.attn_sink_get_device_status() == 0  # read-and-clear
    ref_out = torch.empty_like(out)
    ref_lse = torch.empty_like(lse)
    attn.attn_sink_decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"], ref_out, ref_lse, 0, 0.125, 8,
                          ws)
    torch.cuda.synchronize()
    assert attn.attn_sink_get_device_status() == 0
    import oracle
    ro, rl = oracle.decode(d["q"].cpu(), d["k_cache"].cpu(), d["v_cache"].cpu(), d["seqlens"].cpu(), d["sinks"].cpu(),
                           0, 0.125)
    assert_close_bf16(ref_out, ro, "decode after a timeout")
