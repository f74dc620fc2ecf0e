"""Backward parity at the training shape itself: B=8, L=8192, Hq=64, Hkv=8,
D=64, bf16, dense causal and window-128 layers (fine-tuning through attention,
"GPT-OSS 20B Egitimi: Unsloth, A100 ve Hopper Uyumlulugu", sections 5 and 11).

The GPU runs attn_sink_fwd + attn_sink_bwd on the whole batch.  The fp64
oracle's full backward is too slow for all of it, but the backward is
separable per (batch element, KV group): dq, dk and dv of one slice depend
only on that slice's q, k, v, dout and sinks.  So two full slices -- b = 0 and
b = 7 (whose offsets into q, dout and dq lie past 2^31 bytes) -- are compared
element by element with the oracle's backward of just that slice.

dsink sums -P_sink * D over every row of the batch; the oracle's row
statistics give P_sink and D per row from its own fp64 forward:
  * banded layer: the whole batch, against the full call's dsink;
  * dense layer: batch element 0 (the whole batch would take the oracle
    minutes), against the dsink of a B = 1 call on that element.

This file is collected after the other parity files, so a run that stops at
the first failure has run them already.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from _harness import assert_close_bf16, errors
from gqa_softmax_attention_attn_b200 import attn_sink_bwd, attn_sink_bwd_workspace_size, attn_sink_fwd
from gqa_softmax_attention_attn_b200.inputs import SEEDS, TRAIN, WINDOW, workload_inputs

pytestmark = pytest.mark.gpu

DSINK_REL = 5e-3  # max-abs bound on dsink, relative to its largest entry (plus 1e-5)
SLICES = ((0, 0), (7, 5))  # (batch element, KV group)


@pytest.fixture(scope="module")
def train_inputs():
    return workload_inputs(TRAIN, SEEDS["train"], with_dout=True)


def gpu_fwd_bwd(t, window, scale):
    dev = "cuda"
    q, k, v, s, do = (t[x].to(dev) for x in ("q", "k", "v", "sinks", "dout"))
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, Lq, device=dev, dtype=torch.float32)
    attn_sink_fwd(q, k, v, s, out, lse, window, scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds = torch.empty(Hq, device=dev, dtype=torch.float32)
    ws = torch.empty(attn_sink_bwd_workspace_size(B, Lq, Lk, Hq, Hkv, D, 1), dtype=torch.uint8, device=dev)
    attn_sink_bwd(q, k, v, s, out, do, lse, dq, dk, dv, ds, window, scale, ws)
    torch.cuda.synchronize()
    del q, k, v, do, out, lse, ws
    return dq.cpu(), dk.cpu(), dv.cpu(), ds.cpu()


def check_dsink(got, Dr, Ps, what):
    ref = -(Ps * Dr).sum(axis=(0, 2))
    ma, _ = errors(got, ref)
    bound = DSINK_REL * np.abs(ref).max() + 1e-5
    assert ma <= bound, f"{what}: dsink max_abs={ma:.3e} bound={bound:.3e}"


@pytest.mark.parametrize("window", [0, WINDOW])
def test_train_shape_bwd(train_inputs, window):
    t = train_inputs
    w = TRAIN
    G = w.Hq // w.Hkv
    scale = 1.0 / math.sqrt(w.D)
    dq, dk, dv, ds = gpu_fwd_bwd(t, window, scale)
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all() and torch.isfinite(dv.float()).all()

    for b, g in SLICES:
        hs = slice(g * G, (g + 1) * G)
        rq, rk, rv, _ = oracle.bwd(t["q"][b:b + 1, :, hs], t["k"][b:b + 1, :, g:g + 1], t["v"][b:b + 1, :, g:g + 1],
                                   t["sinks"][hs], t["dout"][b:b + 1, :, hs], window, scale)
        what = f"train b={b} g={g} w={window}"
        assert_close_bf16(dq[b:b + 1, :, hs], rq, f"{what} dq")
        assert_close_bf16(dk[b:b + 1, :, g:g + 1], rk, f"{what} dk")
        assert_close_bf16(dv[b:b + 1, :, g:g + 1], rv, f"{what} dv")

    if window > 0:
        Dr, Ps = oracle.row_stats(t["q"], t["k"], t["v"], t["sinks"], t["dout"], window, scale)
        check_dsink(ds, Dr, Ps, f"train whole batch w={window}")
    else:
        one = {x: t[x][0:1].contiguous() for x in ("q", "k", "v", "dout")}
        one["sinks"] = t["sinks"]
        _, _, _, ds1 = gpu_fwd_bwd(one, window, scale)
        Dr, Ps = oracle.row_stats(one["q"], one["k"], one["v"], one["sinks"], one["dout"], window, scale)
        check_dsink(ds1, Dr, Ps, f"train batch element 0 w={window}")
