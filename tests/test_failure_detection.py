"""Failure detection without a GPU fault: every device-side wait is bounded,
and an expired wait raises a status the host reads, leaving the context usable.

* A self-test kernel waits on an mbarrier that nothing ever arrives on; the
  wait must give up, raise the abort flag and the status bit, and return.
* Through the public API: with the wait limit set to 1 ns, a forward's and a
  decode's waits expire; attn_sink_get_device_status reports
  ATTN_SINK_ERR_TIMEOUT once (and clears it), and the next calls with the
  default limit are correct.
"""
import ctypes
import math

import pytest
import torch

import gqa_softmax_attention_attn_b200 as attn
from _harness import assert_close_bf16
from gqa_softmax_attention_attn_b200 import build
from gqa_softmax_attention_attn_b200.inputs import decode_inputs, prefill_inputs

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


def _with_limit(ns, fn):
    old = attn.attn_sink_set_wait_timeout_ns(ns)
    try:
        fn()
        return attn.attn_sink_get_device_status()
    finally:
        attn.attn_sink_set_wait_timeout_ns(old)


def test_expired_waits_are_reported_and_the_context_stays_usable():
    """With a 1 ns limit every wait that cannot be satisfied at once expires
    (limits below 1 ms poll with a suspend hint of the limit and check the
    clock after every poll).  A forward over the gpt-oss-20b shape has its
    softmax warps wait for the first score tile (a TMA load of Q and K plus
    an MMA) on every CTA, and a decode of long sequences has its consumer warps
    wait for K/V tiles to land, so both must report ATTN_SINK_ERR_TIMEOUT.
    The status is read-and-clear, and the next calls with the default limit
    are correct."""
    import oracle

    dev = "cuda"
    t = prefill_inputs(1, 4096, 4096, 64, 8, 64, torch.bfloat16, 0.5, 1.0, seed=52)
    q, k, v, s = (t[x].to(dev) for x in ("q", "k", "v", "sinks"))
    out = torch.empty_like(q)
    lse = torch.empty(1, 64, 4096, device=dev)
    attn.attn_sink_fwd(q, k, v, s, out, lse, 0, 0.125)  # one-time set-up outside the limit
    assert attn.attn_sink_get_device_status() == 0
    st = _with_limit(1, lambda: attn.attn_sink_fwd(q, k, v, s, out, lse, 0, 0.125))
    assert st == TIMEOUT, f"forward under a 1 ns limit: status {st}"
    assert attn.attn_sink_get_device_status() == 0  # read-and-clear

    d = decode_inputs(4, 16384, 16, 2, 64, 12000, 16384, torch.bfloat16, 0.5, 1.0, seed=51)
    d = {k_: v_.cuda() for k_, v_ in d.items()}
    dout = torch.empty_like(d["q"])
    dlse = torch.empty(4, 16, device=dev)
    ws = torch.empty(max(16, attn.attn_sink_decode_workspace_size(4, 16, 64, 16384, 0, 2)), dtype=torch.uint8,
                     device=dev)
    call = lambda: attn.attn_sink_decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"], dout, dlse,
                                         0, 0.125, 2, ws)
    st = _with_limit(1, call)
    assert st == TIMEOUT, f"decode under a 1 ns limit: status {st}"
    assert attn.attn_sink_get_device_status() == 0

    # the context is usable and the default limit is back: both calls exact again
    attn.attn_sink_fwd(q, k, v, s, out, lse, 0, 0.125)
    call()
    torch.cuda.synchronize()
    assert attn.attn_sink_get_device_status() == 0
    ro, rl = oracle.decode(d["q"].cpu(), d["k_cache"].cpu(), d["v_cache"].cpu(), d["seqlens"].cpu(),
                           d["sinks"].cpu(), 0, 0.125)
    assert_close_bf16(dout, ro, "decode after a timeout")
    rb, rh, ri = (torch.tensor(x, dtype=torch.int32) for x in ([0] * 8, list(range(0, 64, 8)),
                                                                [0, 1, 100, 1000, 2047, 3000, 4000, 4095]))
    fo, fl = oracle.fwd_rows(t["q"], t["k"], t["v"], t["sinks"], rb.numpy(), rh.numpy(), ri.numpy(), 0, 0.125)
    assert_close_bf16(out[0, ri.long(), rh.long()].float().cpu(), fo, "forward after a timeout")
