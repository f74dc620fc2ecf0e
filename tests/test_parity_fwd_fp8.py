"""GPU parity of attn_sink_fwd_fp8 (through the C ABI) against the fp64
oracle on the same e4m3 inputs.

The inputs are the seeded bf16 prefill inputs quantised to e4m3 with one
scale per head (q per query head, k and v per KV head); the oracle widens
every code exactly and applies its scale in fp64 (``oracle.fwd_fp8``), so the
comparison measures the kernel, not the quantisation, at the bf16 forward's
tolerances: the kernel's products of e4m3 values are exact, and P and O are
rounded as in the bf16 forward (P to f16, which is finer than bf16).
"""
import numpy as np
import pytest
import torch

import oracle
from _harness import assert_close_bf16, assert_lse
from gqa_softmax_attention_attn_b200 import attn_sink_fwd_fp8, attn_sink_fwd_fp8_workspace_size
from gqa_softmax_attention_attn_b200.inputs import PREFILL_20B, SEEDS, WINDOW, prefill_inputs, quantize_e4m3_per_head, \
    workload_inputs

pytestmark = pytest.mark.gpu


def quantised(t):
    q8, qs = quantize_e4m3_per_head(t["q"])
    k8, ks = quantize_e4m3_per_head(t["k"])
    v8, vs = quantize_e4m3_per_head(t["v"])
    return {"q8": q8, "k8": k8, "v8": v8, "qs": qs, "ks": ks, "vs": vs, "sinks": t["sinks"]}


def run_fp8(d, window, scale):
    dev = "cuda"
    q8 = d["q8"].to(dev)
    B, Lq, Hq, D = q8.shape
    out = torch.empty(B, Lq, Hq, D, device=dev, dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, Lq, device=dev, dtype=torch.float32)
    Lk, Hkv = d["k8"].shape[1], d["k8"].shape[2]
    ws = torch.full((attn_sink_fwd_fp8_workspace_size(B, Lk, Hkv, D),), 0x7F, dtype=torch.uint8, device=dev)
    attn_sink_fwd_fp8(q8, d["k8"].to(dev), d["v8"].to(dev), d["qs"].to(dev), d["ks"].to(dev), d["vs"].to(dev),
                      d["sinks"].to(dev), out, lse, window, scale, ws)
    torch.cuda.synchronize()
    return out, lse


def oracle_fp8(d, window, scale):
    return oracle.fwd_fp8(d["q8"], d["k8"], d["v8"], d["qs"], d["ks"], d["vs"], d["sinks"], window, scale)


SMALL = [
    # B, Lq, Lk, Hq, Hkv  (ragged tails, Lq != Lk, several GQA group sizes)
    (1, 128, 128, 8, 1),
    (2, 200, 200, 16, 2),
    (1, 77, 300, 8, 8),
    (2, 333, 333, 4, 2),
    (1, 129, 129, 32, 2),
    (3, 64, 64, 24, 3),
]


@pytest.mark.parametrize("window", [0, 1, 5, 128, 100000])
@pytest.mark.parametrize("shape", SMALL)
def test_fp8_small_shapes(shape, window):
    B, Lq, Lk, Hq, Hkv = shape
    t = prefill_inputs(B, Lq, Lk, Hq, Hkv, 64, torch.bfloat16, 0.5, 1.0, seed=hash(shape) % 1000 + window + 7)
    d = quantised(t)
    out, lse = run_fp8(d, window, 0.125)
    ro, rl = oracle_fp8(d, window, 0.125)
    assert_close_bf16(out, ro, f"fp8 out {shape} w={window}")
    assert_lse(lse, rl, f"fp8 lse {shape} w={window}")


def test_fp8_large_logits_force_rescale():
    """Scores far above the sink move the running maximum many times (the
    conditional O rescale path, P up to 2^8 in f16) -- values stay exact."""
    t = prefill_inputs(1, 300, 300, 8, 1, 64, torch.bfloat16, 3.0, 1.0, seed=8)
    d = quantised(t)
    out, lse = run_fp8(d, 0, 0.125)
    ro, rl = oracle_fp8(d, 0, 0.125)
    # the bf16 forward's stress-case bound, for the same reason: |O| up to ~12,
    # where rounding O itself to bf16 (2^-9 relative) already exceeds 2e-2
    assert_close_bf16(out, ro, "fp8 large logits", max_abs=2e-2 * max(1.0, float(np.abs(ro).max()) / 4))
    assert_lse(lse, rl, "fp8 large logits", max_abs=2e-3)


@pytest.mark.parametrize("window", [0, WINDOW])
def test_fp8_prefill_20b_full(window):
    """The gpt-oss-20b prefill (B1 L4096 Hq64 Hkv8), every output element."""
    t = workload_inputs(PREFILL_20B, SEEDS["prefill"])
    d = quantised(t)
    out, lse = run_fp8(d, window, 0.125)
    ro, rl = oracle_fp8(d, window, 0.125)
    assert_close_bf16(out, ro, f"fp8 prefill w={window}")
    assert_lse(lse, rl, f"fp8 prefill w={window}")
