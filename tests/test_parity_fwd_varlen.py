"""GPU parity of attn_sink_fwd_varlen (packed ragged sequences, through the C
ABI) against the fp64 oracle run on each sequence on its own."""
import numpy as np
import pytest
import torch

import oracle
from _harness import assert_close_bf16, assert_lse
from gqa_softmax_attention_attn_b200 import attn_sink_fwd_varlen
from gqa_softmax_attention_attn_b200.inputs import WINDOW, prefill_inputs

pytestmark = pytest.mark.gpu


def packed(lens_q, lens_k, Hq, Hkv, seed):
    total_q, total_k = sum(lens_q), sum(lens_k)
    t = prefill_inputs(1, total_q, total_k, Hq, Hkv, 64, torch.bfloat16, 0.5, 1.0, seed=seed)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    return {"q": t["q"][0], "k": t["k"][0], "v": t["v"][0], "sinks": t["sinks"], "cu_q": cu_q, "cu_k": cu_k}


def run_varlen(d, window, scale):
    dev = "cuda"
    q, k, v, s = (d[x].to(dev) for x in ("q", "k", "v", "sinks"))
    total_q, Hq, _ = q.shape
    out = torch.full_like(q, float("nan"))
    lse = torch.full((Hq, total_q), float("nan"), device=dev)
    cu_q = torch.from_numpy(d["cu_q"]).to(dev)
    cu_k = torch.from_numpy(d["cu_k"]).to(dev)
    max_q = int(np.diff(d["cu_q"]).max())
    attn_sink_fwd_varlen(q, k, v, s, out, lse, cu_q, cu_k, max_q, window, scale)
    torch.cuda.synchronize()
    return out, lse


CASES = {
    # sequence lengths: ragged, with single tokens, a tile edge, and an empty sequence
    "ragged": ([1, 17, 300, 129, 0, 64, 1000], None),
    # chunked prefill: every sequence has a cached prefix (keys before its first query)
    "prefix": ([16, 200, 1, 77], [40, 200, 513, 300]),
}


@pytest.mark.parametrize("window", [0, 5, WINDOW])
@pytest.mark.parametrize("heads", [(64, 8), (16, 2), (8, 8)])
@pytest.mark.parametrize("case", sorted(CASES))
def test_varlen_matches_each_sequence(case, heads, window):
    lq, lk = CASES[case]
    lk = lk or lq
    Hq, Hkv = heads
    d = packed(lq, lk, Hq, Hkv, seed=101 + Hq + window + len(case))
    out, lse = run_varlen(d, window, 0.125)
    ro, rl = oracle.fwd_varlen(d["q"], d["k"], d["v"], d["sinks"], d["cu_q"], d["cu_k"], window, 0.125)
    assert_close_bf16(out, ro, f"varlen {case} heads={heads} w={window}")
    assert_lse(lse, rl, f"varlen {case} heads={heads} w={window}")


def test_varlen_disaggregated_prefill_batch():
    """A prefill batch of mixed lengths as a prefill server receives it: 12
    sequences with seeded lengths in [256, 4096], gpt-oss-20b heads, dense and
    window-128 layers, every output element."""
    g = np.random.default_rng(1002)
    lens = [int(x) for x in g.integers(256, 4097, 12)]
    d = packed(lens, lens, 64, 8, seed=1102)
    for window in (0, WINDOW):
        out, lse = run_varlen(d, window, 0.125)
        ro, rl = oracle.fwd_varlen(d["q"], d["k"], d["v"], d["sinks"], d["cu_q"], d["cu_k"], window, 0.125)
        assert_close_bf16(out, ro, f"varlen batch w={window}")
        assert_lse(lse, rl, f"varlen batch w={window}")
