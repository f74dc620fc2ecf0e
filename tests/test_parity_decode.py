"""GPU parity of attn_sink_decode (through the C ABI) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from _harness import assert_close_bf16, assert_close_fp32, assert_lse
from gqa_softmax_attention_attn_b200 import attn_sink_decode, attn_sink_decode_workspace_size
from gqa_softmax_attention_attn_b200.inputs import DECODE, SEEDS, WINDOW, decode_inputs

pytestmark = pytest.mark.gpu


def run_decode(d, window, scale, num_splits=0):
    dev = "cuda"
    q = d["q"].to(dev)
    kc, vc = d["k_cache"].to(dev), d["v_cache"].to(dev)
    sl, s = d["seqlens"].to(dev), d["sinks"].to(dev)
    B, Hq, D = q.shape
    Lmax = kc.shape[1]
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, device=dev, dtype=torch.float32)
    nbytes = attn_sink_decode_workspace_size(B, Hq, D, Lmax, window, num_splits)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    attn_sink_decode(q, kc, vc, sl, s, out, lse, window, scale, num_splits, ws)
    torch.cuda.synchronize()
    return out, lse


_cache = {}


def _full_inputs():
    if "inputs" not in _cache:
        w = DECODE
        _cache["inputs"] = decode_inputs(w.B, w.Lmax, w.Hq, w.Hkv, w.D, w.len_lo, w.len_hi, w.dtype, w.qkv_std,
                                         w.sink_std, seed=SEEDS["decode"])
    return _cache["inputs"]


def _oracle_full(window, scale):
    """Oracle per sequence on its own prefix (keeps fp64 copies small)."""
    key = (window, scale)
    if key not in _cache:
        d = _full_inputs()
        outs, lses = [], []
        for b in range(d["q"].shape[0]):
            L = int(d["seqlens"][b])
            o, l = oracle.decode(d["q"][b:b + 1], d["k_cache"][b:b + 1, :L], d["v_cache"][b:b + 1, :L],
                                 d["seqlens"][b:b + 1], d["sinks"], window, scale)
            outs.append(o)
            lses.append(l)
        _cache[key] = (np.concatenate(outs), np.concatenate(lses))
    return _cache[key]


@pytest.mark.parametrize("window", [0, WINDOW])
@pytest.mark.parametrize("splits", [0, 1, 4, 8, 16, 32])
def test_decode_full_workload(window, splits):
    """64 sequences, lengths ~ U[1024, 32768], every output element, dense and window-128."""
    if "dev" not in _cache:
        _cache["dev"] = {k: v.cuda() for k, v in _full_inputs().items()}
    scale = 1.0 / math.sqrt(DECODE.D)
    out, lse = run_decode(_cache["dev"], window, scale, splits)
    ro, rl = _oracle_full(window, scale)
    assert_close_bf16(out, ro, f"decode w={window} splits={splits}")
    assert_lse(lse, rl, f"decode w={window} splits={splits}")


def test_split_count_invariance():
    """The sink is counted once whatever the split count: results for 1..32
    splits agree with each other far inside the bf16 tolerance."""
    d = decode_inputs(8, 4096, 16, 2, 64, 1, 4096, torch.bfloat16, 0.5, 1.0, seed=21)
    outs = [run_decode(d, 0, 0.125, s) for s in (1, 2, 4, 8, 16, 32)]
    for o, l in outs[1:]:
        assert (o.float() - outs[0][0].float()).abs().max().item() < 4e-3
        assert (l - outs[0][1]).abs().max().item() < 1e-4


@pytest.mark.parametrize("window", [0, 3, 64, 128])
def test_decode_edges_bf16(window):
    """Lengths 1, Lmax and values around chunk and window edges; group sizes 4 and 16."""
    for (Hq, Hkv) in ((16, 4), (32, 2), (8, 8)):
        d = decode_inputs(9, 700, Hq, Hkv, 64, 1, 700, torch.bfloat16, 0.5, 1.0, seed=22 + Hq)
        d["seqlens"] = torch.tensor([1, 700, 64, 65, 127, 128, 129, 2, 699], dtype=torch.int32)
        for splits in (0, 3, 11):
            out, lse = run_decode(d, window, 0.125, splits)
            ro, rl = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"], window, 0.125)
            assert_close_bf16(out, ro, f"edges Hq={Hq} Hkv={Hkv} w={window} s={splits}")
            assert_lse(lse, rl, f"edges Hq={Hq} Hkv={Hkv} w={window} s={splits}")


@pytest.mark.parametrize("window,splits", [(160, 0), (192, 0), (192, 1), (0, 8)])
def test_decode_short_splits(window, splits):
    """Splits of at most 192 keys run with a three-stage ring: windows of 160
    and 192 keys and dense splits of 188 keys span up to four 64-key tiles, so
    the ring wraps within a split."""
    d = decode_inputs(9, 1500, 16, 2, 64, 1, 1500, torch.bfloat16, 0.5, 1.0, seed=29 + window + splits)
    d["seqlens"] = torch.tensor([1, 1500, 191, 192, 193, 255, 256, 257, 1023], dtype=torch.int32)
    out, lse = run_decode(d, window, 0.125, splits)
    ro, rl = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"], window, 0.125)
    assert_close_bf16(out, ro, f"short splits w={window} s={splits}")
    assert_lse(lse, rl, f"short splits w={window} s={splits}")


@pytest.mark.parametrize("window", [0, 128])
def test_decode_fp32_exact(window):
    d = decode_inputs(4, 600, 8, 2, 64, 1, 600, torch.float32, 1.0, 1.0, seed=23)
    for splits in (0, 1, 5):
        out, lse = run_decode(d, window, 0.125, splits)
        ro, rl = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"], window, 0.125)
        assert_close_fp32(out, ro, "decode fp32")
        assert_close_fp32(lse, rl, "decode fp32 lse")


def test_decode_matches_last_prefill_row():
    """Decode for sequence b equals row len_b - 1 of a prefill over that prefix
    (two different kernels; both against the same oracle row)."""
    from gqa_softmax_attention_attn_b200 import attn_sink_fwd

    d = decode_inputs(3, 1000, 16, 2, 64, 100, 1000, torch.bfloat16, 0.5, 1.0, seed=24)
    out, lse = run_decode(d, 0, 0.125, 4)
    for b in range(3):
        L = int(d["seqlens"][b])
        q = torch.zeros(1, L, 16, 64, dtype=torch.bfloat16)
        q[0, L - 1] = d["q"][b]
        k = d["k_cache"][b:b + 1, :L].contiguous().cuda()
        v = d["v_cache"][b:b + 1, :L].contiguous().cuda()
        po = torch.empty(1, L, 16, 64, dtype=torch.bfloat16, device="cuda")
        pl = torch.empty(1, 16, L, dtype=torch.float32, device="cuda")
        attn_sink_fwd(q.cuda(), k, v, d["sinks"].cuda(), po, pl, 0, 0.125)
        torch.cuda.synchronize()
        assert (po[0, L - 1].float() - out[b].float()).abs().max().item() < 1e-2
        assert (pl[0, :, L - 1] - lse[b]).abs().max().item() < 1e-3
