"""GPU parity of attn_sink_fwd (through the C ABI) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from _harness import assert_close_bf16, assert_close_fp32, assert_lse, errors
import gqa_softmax_attention_attn_b200 as attn
from gqa_softmax_attention_attn_b200 import attn_sink_fwd
from gqa_softmax_attention_attn_b200.inputs import (LONG_BANDED, LONG_DENSE, PREFILL_20B, SEEDS, TINY_FP32, TRAIN,
                                                    WINDOW, prefill_inputs, sample_rows, workload_inputs)

pytestmark = pytest.mark.gpu


def run_fwd(t, window, scale):
    dev = "cuda"
    q, k, v = t["q"].to(dev), t["k"].to(dev), t["v"].to(dev)
    s = t["sinks"].to(dev)
    B, Lq, Hq, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, Lq, device=dev, dtype=torch.float32)
    attn_sink_fwd(q, k, v, s, out, lse, window, scale)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("window", [0, WINDOW])
def test_tiny_fp32_exact(window):
    w = TINY_FP32
    t = workload_inputs(w, SEEDS["tiny"])
    scale = 1.0 / math.sqrt(w.D)
    out, lse = run_fwd(t, window, scale)
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, scale)
    assert_close_fp32(out, ro, "out")
    assert_close_fp32(lse, rl, "lse")


SMALL = [
    # B, Lq, Lk, Hq, Hkv  (ragged tails, Lq != Lk, several GQA group sizes)
    (1, 128, 128, 8, 1),
    (2, 200, 200, 16, 2),
    (1, 77, 300, 8, 8),
    (2, 333, 333, 4, 2),
    (1, 129, 129, 32, 2),
    (1, 50, 40, 8, 1),
    (3, 64, 64, 24, 3),
]


@pytest.mark.parametrize("window", [0, 1, 5, 128, 100000])
@pytest.mark.parametrize("shape", SMALL)
def test_bf16_small_shapes(shape, window):
    B, Lq, Lk, Hq, Hkv = shape
    t = prefill_inputs(B, Lq, Lk, Hq, Hkv, 64, torch.bfloat16, 0.5, 1.0, seed=hash(shape) % 1000 + window)
    scale = 0.125
    out, lse = run_fwd(t, window, scale)
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, scale)
    assert_close_bf16(out, ro, f"out {shape} w={window}")
    assert_lse(lse, rl, f"lse {shape} w={window}")


@pytest.mark.parametrize("window", [0, 128])
def test_bf16_many_heads(window):
    """1040 query heads in groups of 8 (130 KV heads): a wide head dimension of
    the grid for both forward kernels."""
    t = prefill_inputs(1, 40, 40, 1040, 130, 64, torch.bfloat16, 0.5, 1.0, seed=41 + window)
    out, lse = run_fwd(t, window, 0.125)
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, 0.125)
    assert_close_bf16(out, ro, f"1040 heads w={window}")
    assert_lse(lse, rl, f"1040 heads w={window}")


@pytest.mark.parametrize("sink", [float("-inf"), 50.0, -30.0])
def test_bf16_extreme_sinks(sink):
    t = prefill_inputs(1, 150, 150, 16, 2, 64, torch.bfloat16, 0.5, 1.0, seed=7, sink_fill=sink)
    out, lse = run_fwd(t, 0, 0.125)
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, 0.125)
    assert_close_bf16(out, ro, f"sink={sink}")
    assert_lse(lse, rl, f"sink={sink}")
    assert torch.isfinite(out).all()


def test_bf16_large_logits_force_rescale():
    """Scores far above the sink move the running maximum many times (the
    conditional O rescale path) -- values stay exact."""
    t = prefill_inputs(1, 300, 300, 8, 1, 64, torch.bfloat16, 3.0, 1.0, seed=8)
    out, lse = run_fwd(t, 0, 0.125)
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, 0.125)
    # Inputs with std 3 give |O| up to ~12, where rounding O itself to bf16
    # (2^-9 relative) already exceeds 2e-2: the bound scales with max|O| here.
    assert_close_bf16(out, ro, "large logits", max_abs=2e-2 * max(1.0, float(np.abs(ro).max()) / 4))
    assert_lse(lse, rl, "large logits", max_abs=2e-3)


def test_rows_without_keys_and_neg_inf_sink():
    t = prefill_inputs(1, 100, 20, 8, 2, 64, torch.bfloat16, 0.5, 1.0, seed=9)
    t["sinks"][:4] = float("-inf")
    out, lse = run_fwd(t, 0, 0.125)
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, 0.125)
    assert_close_bf16(out, ro, "no keys")
    lg = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(lg), np.isneginf(rl))
    assert_lse(lse, rl, "no keys")


@pytest.mark.parametrize("window", [0, WINDOW])
def test_prefill_20b_full(window):
    """gpt-oss-20b shaped prefill (B1 L4096 Hq64 Hkv8), every output element."""
    w = PREFILL_20B
    t = workload_inputs(w, SEEDS["prefill"])
    scale = 1.0 / math.sqrt(w.D)
    out, lse = run_fwd(t, window, scale)
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, scale)
    ma, rel = assert_close_bf16(out, ro, f"prefill w={window}")
    assert_lse(lse, rl, f"prefill w={window}")


def _sampled(w, seed, window, n=64):
    t = workload_inputs(w, seed)
    scale = 1.0 / math.sqrt(w.D)
    out, lse = run_fwd(t, window, scale)
    rb, rh, ri = sample_rows(w.B, w.Hq, w.L, n, seed + 17, window, sinks=t["sinks"])
    ro, rl = oracle.fwd_rows(t["q"], t["k"], t["v"], t["sinks"], rb.numpy(), rh.numpy(), ri.numpy(), window, scale)
    go = out[rb.long(), ri.long(), rh.long()].float().cpu()
    gl = lse[rb.long(), rh.long(), ri.long()].cpu()
    assert_close_bf16(go, ro, f"{w.name} w={window} sampled")
    assert_lse(gl, rl, f"{w.name} w={window} sampled")
    # properties that hold at any size: finite, and |O| <= max|v| (convex combination scaled by < 1)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    assert out.abs().max().item() <= t["v"].abs().max().item() + 1e-2


@pytest.mark.parametrize("window", [0, WINDOW])
def test_train_shape_sampled(window):
    _sampled(TRAIN, SEEDS["train"], window)


def test_long_banded_sampled():
    _sampled(LONG_BANDED, SEEDS["long"], WINDOW)


def test_long_dense_sampled():
    _sampled(LONG_DENSE, SEEDS["long"], 0)


def test_deterministic_and_stream_ordered():
    t = prefill_inputs(1, 512, 512, 64, 8, 64, torch.bfloat16, 0.5, 1.0, seed=11)
    o1, l1 = run_fwd(t, 0, 0.125)
    o2, l2 = run_fwd(t, 0, 0.125)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_graph_replay_and_concurrent_streams():
    # running CTAs take over the items of CTAs that have not started yet
    # (cluster launch control): replaying a captured launch, and launches of
    # both layer types running at once on two streams, must still each process
    # every item exactly once
    t = prefill_inputs(1, 2048, 2048, 64, 8, 64, torch.bfloat16, 0.5, 1.0, seed=12)
    dev = "cuda"
    q, k, v, s = (t[x].to(dev) for x in ("q", "k", "v", "sinks"))
    refs = {w: run_fwd(t, w, 0.125) for w in (0, WINDOW)}
    out = torch.empty_like(q)
    lse = torch.empty(1, 64, 2048, device=dev)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        attn_sink_fwd(q, k, v, s, out, lse, 0, 0.125, stream)  # outside the capture: one-time set-up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        attn_sink_fwd(q, k, v, s, out, lse, 0, 0.125, stream)
    for _ in range(3):
        out.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, refs[0][0]) and torch.equal(lse, refs[0][1])
    del g
    # two streams, dense launches on one and window-128 launches on the other,
    # overlapping on the device
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = [(torch.empty_like(q), torch.empty_like(lse)) for _ in range(8)]
    torch.cuda.synchronize()
    for i, (o, l) in enumerate(outs):
        st, w = (s1, 0) if i % 2 == 0 else (s2, WINDOW)
        with torch.cuda.stream(st):
            attn_sink_fwd(q, k, v, s, o, l, w, 0.125, st)
    torch.cuda.synchronize()
    for i, (o, l) in enumerate(outs):
        ro, rl = refs[0 if i % 2 == 0 else WINDOW]
        assert torch.equal(o, ro) and torch.equal(l, rl), f"launch {i}"
    assert attn.attn_sink_get_device_status() == 0


def test_concurrent_replays_of_two_graphs():
    """Two captured forwards (a dense and a banded layer) replayed at the same
    time on two streams, many times: every replay complete and exact."""
    t = prefill_inputs(1, 1024, 1024, 64, 8, 64, torch.bfloat16, 0.5, 1.0, seed=13)
    dev = "cuda"
    q, k, v, s = (t[x].to(dev) for x in ("q", "k", "v", "sinks"))
    refs = {w: run_fwd(t, w, 0.125) for w in (0, WINDOW)}
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    bufs, graphs = {}, {}
    for w, st in ((0, s1), (WINDOW, s2)):
        bufs[w] = (torch.empty_like(q), torch.empty(1, 64, 1024, device=dev))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st, capture_error_mode="thread_local"):
            attn_sink_fwd(q, k, v, s, bufs[w][0], bufs[w][1], w, 0.125, st)
        graphs[w] = (g, st)
    for _ in range(10):
        for w in (0, WINDOW):
            bufs[w][0].zero_()
            bufs[w][1].zero_()
        torch.cuda.synchronize()
        for w in (0, WINDOW):
            g, st = graphs[w]
            with torch.cuda.stream(st):
                g.replay()
        torch.cuda.synchronize()
        for w in (0, WINDOW):
            assert torch.equal(bufs[w][0], refs[w][0]) and torch.equal(bufs[w][1], refs[w][1])
    del graphs
    assert attn.attn_sink_get_device_status() == 0
