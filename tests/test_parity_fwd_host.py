"""GPU parity of attn_sink_fwd_host (inputs and outputs in host memory, the
transfers overlapped with the computation chunk by chunk) through the C ABI:
bit for bit against attn_sink_fwd on the same inputs (the chunks hold whole
work items of the forward), and against the fp64 oracle."""
import pytest
import torch

import oracle
from _harness import assert_close_bf16, assert_lse
from gqa_softmax_attention_attn_b200 import attn_sink_fwd, attn_sink_fwd_host, attn_sink_fwd_host_workspace_size
from gqa_softmax_attention_attn_b200.inputs import prefill_inputs

pytestmark = pytest.mark.gpu

SCALE = 0.125


def host_call(t, window, chunks, pin=True):
    q, k, v, s = (t[x].contiguous() for x in ("q", "k", "v", "sinks"))
    if pin:
        q, k, v, s = (x.pin_memory() for x in (q, k, v, s))
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, Lq), float("nan"), dtype=torch.float32)
    if pin:
        out, lse = out.pin_memory(), lse.pin_memory()
    ws = torch.full((attn_sink_fwd_host_workspace_size(B, Lq, Lk, Hq, Hkv, D),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    attn_sink_fwd_host(q, k, v, s, out, lse, window, SCALE, ws, chunks)
    torch.cuda.synchronize()
    return out, lse


def device_call(t, window):
    q, k, v, s = (t[x].cuda() for x in ("q", "k", "v", "sinks"))
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[2], q.shape[1], device="cuda", dtype=torch.float32)
    attn_sink_fwd(q, k, v, s, out, lse, window, SCALE)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("window", [0, 128])
@pytest.mark.parametrize("shape,chunks", [((2, 1000, 1000, 16, 2), 3), ((1, 700, 900, 8, 1), 8),
                                          ((1, 256, 256, 64, 8), 1), ((2, 640, 640, 4, 1), 5),
                                          ((3, 129, 200, 8, 8), 64)])
def test_host_equals_device(shape, chunks, window):
    """Group sizes 1-8 (items of 16 to 128 positions), Lq < Lk, ragged last
    chunks, one chunk and more chunks than 128-position blocks."""
    B, Lq, Lk, Hq, Hkv = shape
    t = prefill_inputs(B, Lq, Lk, Hq, Hkv, 64, torch.bfloat16, 0.5, 1.0, 0.1, seed=90 + Lq + window)
    o1, l1 = host_call(t, window, chunks)
    o2, l2 = device_call(t, window)
    assert torch.equal(o1, o2), f"out differs: {shape} chunks={chunks} w={window}"
    assert torch.equal(l1, l2), f"lse differs: {shape} chunks={chunks} w={window}"


def test_pageable_host_memory():
    """Unpinned host buffers: the copies do not overlap, the results are the same."""
    t = prefill_inputs(1, 600, 600, 16, 2, 64, torch.bfloat16, 0.5, 1.0, 0.1, seed=97)
    o1, l1 = host_call(t, 128, 4, pin=False)
    o2, l2 = device_call(t, 128)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("window", [0, 128])
def test_host_against_oracle(window):
    t = prefill_inputs(1, 300, 300, 8, 1, 64, torch.bfloat16, 0.5, 1.0, 0.1, seed=98 + window)
    out, lse = host_call(t, window, 4)
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, SCALE)
    assert_close_bf16(out, ro, f"host fwd w={window}")
    assert_lse(lse, rl, f"host fwd w={window}")


@pytest.mark.parametrize("chunks", [4, 8])
@pytest.mark.parametrize("window", [0, 128])
def test_host_prefill_20b(window, chunks):
    """The gpt-oss-20b prefill (B1 L4096 Hq64 Hkv8), bit for bit: four chunks
    (640, 1408, 1408, 640 positions: the end chunks take half the others') and
    eight."""
    t = prefill_inputs(1, 4096, 4096, 64, 8, 64, torch.bfloat16, 0.5, 1.0, 0.1, seed=99 + window)
    o1, l1 = host_call(t, window, chunks)
    o2, l2 = device_call(t, window)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
