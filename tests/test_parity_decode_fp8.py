"""GPU parity of attn_sink_decode_fp8 (through the C ABI) against the fp64
oracle on the same e4m3 caches.

The caches are the seeded bf16 decode caches quantised to e4m3 with one scale
per KV head (the input format); the oracle widens every code exactly and
multiplies by its scale in fp64 (``oracle.decode_fp8``), so the comparison
measures the kernel, not the quantisation.  Cache rows beyond each sequence's
length are filled with the NaN code 0x7f: they must never reach the output.
"""
import numpy as np
import pytest
import torch

import oracle
from _harness import assert_close_bf16, assert_lse
from gqa_softmax_attention_attn_b200 import attn_sink_decode_fp8, attn_sink_decode_workspace_size
from gqa_softmax_attention_attn_b200.inputs import DECODE, SEEDS, WINDOW, decode_inputs, quantize_e4m3_per_head

pytestmark = pytest.mark.gpu

NAN_CODE = 0x7F


def fp8_inputs(B, Lmax, Hq, Hkv, len_lo, len_hi, seed, poison=True):
    d = decode_inputs(B, Lmax, Hq, Hkv, 64, len_lo, len_hi, torch.bfloat16, 0.5, 1.0, seed=seed)
    k8, ks = quantize_e4m3_per_head(d["k_cache"])
    v8, vs = quantize_e4m3_per_head(d["v_cache"])
    if poison:
        for b, L in enumerate(d["seqlens"].tolist()):
            k8[b, L:] = NAN_CODE
            v8[b, L:] = NAN_CODE
    return {"q": d["q"], "k8": k8, "v8": v8, "ks": ks, "vs": vs, "seqlens": d["seqlens"], "sinks": d["sinks"]}


def run_fp8(d, window, scale, num_splits=0):
    dev = "cuda"
    q = d["q"].to(dev)
    B, Hq, D = q.shape
    Lmax = d["k8"].shape[1]
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, device=dev, dtype=torch.float32)
    nbytes = attn_sink_decode_workspace_size(B, Hq, D, Lmax, window, num_splits)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    attn_sink_decode_fp8(q, d["k8"].to(dev), d["v8"].to(dev), d["ks"].to(dev), d["vs"].to(dev),
                         d["seqlens"].to(dev), d["sinks"].to(dev), out, lse, window, scale, num_splits, ws)
    torch.cuda.synchronize()
    return out, lse


def oracle_fp8(d, window, scale):
    """Per sequence on its own prefix (small fp64 copies; no poisoned row is read)."""
    outs, lses = [], []
    for b in range(d["q"].shape[0]):
        L = int(d["seqlens"][b])
        o, l = oracle.decode_fp8(d["q"][b:b + 1], d["k8"][b:b + 1, :L], d["v8"][b:b + 1, :L], d["ks"], d["vs"],
                                 d["seqlens"][b:b + 1], d["sinks"], window, scale)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs), np.concatenate(lses)


@pytest.mark.parametrize("window", [0, 3, WINDOW])
@pytest.mark.parametrize("splits", [0, 1, 5])
@pytest.mark.parametrize("heads", [(16, 2), (8, 8), (32, 2)])
def test_fp8_small(window, splits, heads):
    Hq, Hkv = heads
    d = fp8_inputs(5, 1500, Hq, Hkv, 1, 1500, seed=61 + Hq + window)
    out, lse = run_fp8(d, window, 0.125, splits)
    ro, rl = oracle_fp8(d, window, 0.125)
    assert_close_bf16(out, ro, f"fp8 decode w={window} splits={splits} heads={heads}")
    assert_lse(lse, rl, f"fp8 decode w={window} splits={splits} heads={heads}")


_cache = {}


def _workload():
    if "d" not in _cache:
        w = DECODE
        _cache["d"] = fp8_inputs(w.B, w.Lmax, w.Hq, w.Hkv, w.len_lo, w.len_hi, SEEDS["decode"])
    return _cache["d"]


@pytest.mark.parametrize("window,splits", [(200, 0), (256, 0), (0, 6)])
def test_fp8_short_splits(window, splits):
    """Splits of at most 256 keys run with a two-stage ring (four CTAs per
    SM): windows of 200 and 256 keys and dense splits of 250 keys span up to
    three 128-key tiles, so the ring wraps within a split."""
    d = fp8_inputs(9, 1500, 16, 2, 1, 1500, seed=71 + window + splits)
    out, lse = run_fp8(d, window, 0.125, splits)
    ro, rl = oracle_fp8(d, window, 0.125)
    assert_close_bf16(out, ro, f"fp8 short splits w={window} s={splits}")
    assert_lse(lse, rl, f"fp8 short splits w={window} s={splits}")


@pytest.mark.parametrize("window", [0, WINDOW])
def test_fp8_decode_workload_full(window):
    """The 64-sequence decode workload (lengths U[1024, 32768], Hq64 Hkv8) with
    e4m3 caches: every output element, automatic and fixed split counts."""
    d = _workload()
    scale = 1.0 / 8.0
    ro, rl = oracle_fp8(d, window, scale)
    for splits in (0, 8, 32):
        out, lse = run_fp8(d, window, scale, splits)
        assert_close_bf16(out, ro, f"fp8 workload w={window} splits={splits}")
        assert_lse(lse, rl, f"fp8 workload w={window} splits={splits}")
        assert torch.isfinite(out.float()).all()


def test_fp8_split_count_invariance():
    d = fp8_inputs(4, 8192, 16, 2, 100, 8192, seed=71)
    ref, _ = run_fp8(d, 0, 0.125, 1)
    for splits in (2, 4, 16, 32):
        out, _ = run_fp8(d, 0, 0.125, splits)
        assert (out.float() - ref.float()).abs().max().item() <= 1e-2
