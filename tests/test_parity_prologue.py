"""GPU parity of attn_sink_qkv_prologue (bias + YaRN rotary embedding + split,
through the C ABI) against the fp64 oracle: alone, appending to a decode
cache, and chained into the prefill forward."""
import numpy as np
import pytest
import torch

import oracle
from _harness import assert_close_bf16, assert_lse
from gqa_softmax_attention_attn_b200 import attn_sink_fwd, attn_sink_qkv_prologue
from gqa_softmax_attention_attn_b200.inputs import WINDOW

pytestmark = pytest.mark.gpu

# the gpt-oss context extension: 4096 original positions scaled 32x to 131072
YARN = dict(rope_theta=150000.0, rope_factor=32.0, rope_original_max_pos=4096, beta_fast=32.0, beta_slow=1.0)
ORACLE_YARN = dict(base=150000.0, factor=32.0, original_max_pos=4096, beta_fast=32.0, beta_slow=1.0)
PLAIN = dict(rope_theta=10000.0, rope_factor=1.0)
ORACLE_PLAIN = dict(base=10000.0, factor=1.0)


def make_qkv(T, Hq, Hkv, seed, max_pos):
    g = torch.Generator().manual_seed(seed)
    qkv = (torch.randn(T, (Hq + 2 * Hkv) * 64, generator=g) * 0.5).to(torch.bfloat16)
    bias = torch.randn((Hq + 2 * Hkv) * 64, generator=g) * 0.1
    pos = torch.randint(0, max_pos, (T,), generator=g, dtype=torch.int64).to(torch.int32)
    return qkv, bias, pos


@pytest.mark.parametrize("interleaved", [False, True])
@pytest.mark.parametrize("rope", ["yarn", "plain"])
@pytest.mark.parametrize("with_bias", [True, False])
def test_prologue_matches_oracle(interleaved, rope, with_bias):
    T, Hq, Hkv = 333, 64, 8
    qkv, bias, pos = make_qkv(T, Hq, Hkv, seed=201 + interleaved, max_pos=131072)
    kw, okw = (YARN, ORACLE_YARN) if rope == "yarn" else (PLAIN, ORACLE_PLAIN)
    dev = "cuda"
    q = torch.empty(T, Hq, 64, dtype=torch.bfloat16, device=dev)
    k = torch.empty(T, Hkv, 64, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    attn_sink_qkv_prologue(qkv.to(dev), bias.to(dev) if with_bias else None, pos.to(dev), q, k, v,
                           interleaved=interleaved, **kw)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_prologue(qkv, bias if with_bias else None, pos, Hq, Hkv, 64, interleaved=interleaved,
                                     **okw)
    assert_close_bf16(q, rq, f"q {rope} interleaved={interleaved}")
    assert_close_bf16(k, rk, f"k {rope} interleaved={interleaved}")
    assert_close_bf16(v, rv, f"v {rope} interleaved={interleaved}")


@pytest.mark.parametrize("shape", [(9, 8, 1), (7, 300, 4), (5, 600, 8), (3, 784, 8), (130, 4, 4)])
def test_prologue_row_widths(shape):
    """Narrow and very wide rows (10 to 800 heads), token counts that leave
    the last 8-token CTA ragged."""
    T, Hq, Hkv = shape
    qkv, bias, pos = make_qkv(T, Hq, Hkv, seed=221 + Hq, max_pos=131072)
    dev = "cuda"
    q = torch.empty(T, Hq, 64, dtype=torch.bfloat16, device=dev)
    k = torch.empty(T, Hkv, 64, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    attn_sink_qkv_prologue(qkv.to(dev), bias.to(dev), pos.to(dev), q, k, v, **YARN)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_prologue(qkv, bias, pos, Hq, Hkv, 64, **ORACLE_YARN)
    assert_close_bf16(q, rq, f"q {shape}")
    assert_close_bf16(k, rk, f"k {shape}")
    assert_close_bf16(v, rv, f"v {shape}")


def test_prologue_appends_to_a_decode_cache():
    """kv_rows sends token t's k and v to row b * Lmax + p of a [B, Lmax] cache;
    every other row keeps its contents, and rows outside the cache are skipped."""
    B, Lmax, Hq, Hkv = 4, 100, 16, 2
    qkv, bias, _ = make_qkv(B, Hq, Hkv, seed=211, max_pos=Lmax)
    pos = torch.tensor([0, 57, 99, 13], dtype=torch.int32)
    dev = "cuda"
    kc = torch.full((B * Lmax, Hkv, 64), 7.0, dtype=torch.bfloat16, device=dev)
    vc = torch.full_like(kc, -3.0)
    rows = (torch.arange(B, dtype=torch.int32) * Lmax + pos)
    rows_dev = rows.clone()
    rows_dev[3] = B * Lmax + 5  # outside the cache: not written
    q = torch.empty(B, Hq, 64, dtype=torch.bfloat16, device=dev)
    attn_sink_qkv_prologue(qkv.to(dev), bias.to(dev), pos.to(dev), q, kc, vc, kv_rows=rows_dev.to(dev), **YARN)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_prologue(qkv, bias, pos, Hq, Hkv, 64, **ORACLE_YARN)
    assert_close_bf16(q, rq, "q")
    assert_close_bf16(kc[rows[:3].long()], rk[:3], "k rows")
    assert_close_bf16(vc[rows[:3].long()], rv[:3], "v rows")
    untouched = torch.ones(B * Lmax, dtype=torch.bool)
    untouched[rows[:3].long()] = False
    assert (kc[untouched.to(dev)] == 7.0).all() and (vc[untouched.to(dev)] == -3.0).all()


@pytest.mark.parametrize("window", [0, WINDOW])
def test_prologue_then_prefill_forward(window):
    """The prologue and the forward chained on one sequence of 700 tokens at
    positions 0..699, against the oracle's prologue fed to the oracle's
    forward.  The prologue's outputs are bf16 by definition of the call, so
    the oracle's fp64 prologue outputs are rounded to bf16 (round to nearest
    even) before its forward, as the GPU's are."""
    T, Hq, Hkv = 700, 64, 8
    qkv, bias, _ = make_qkv(T, Hq, Hkv, seed=221, max_pos=T)
    pos = torch.arange(T, dtype=torch.int32)
    dev = "cuda"
    q = torch.empty(1, T, Hq, 64, dtype=torch.bfloat16, device=dev)
    k = torch.empty(1, T, Hkv, 64, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    attn_sink_qkv_prologue(qkv.to(dev), bias.to(dev), pos.to(dev), q[0], k[0], v[0], **YARN)
    sinks = torch.randn(Hq, generator=torch.Generator().manual_seed(222))
    out = torch.empty_like(q)
    lse = torch.empty(1, Hq, T, device=dev)
    attn_sink_fwd(q, k, v, sinks.to(dev), out, lse, window, 0.125)
    torch.cuda.synchronize()
    rq, rk, rv = (torch.from_numpy(x).to(torch.bfloat16)[None]
                  for x in oracle.qkv_prologue(qkv, bias, pos, Hq, Hkv, 64, **ORACLE_YARN))
    ro, rl = oracle.fwd(rq, rk, rv, sinks, window, 0.125)
    assert_close_bf16(out, ro, f"prologue + forward w={window}")
    assert_lse(lse, rl, f"prologue + forward w={window}")
