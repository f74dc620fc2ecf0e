"""GPU parity of attn_sink_decode_paged (through the C ABI): against the fp64
oracle on the same keys and values, and bit for bit against the contiguous
decode where both cut the keys into the same tiles."""
import math

import numpy as np
import pytest
import torch

import oracle
from _harness import assert_close_bf16, assert_lse
from gqa_softmax_attention_attn_b200 import (attn_sink_decode, attn_sink_decode_paged,
                                             attn_sink_decode_paged_workspace_size, attn_sink_decode_workspace_size)
from gqa_softmax_attention_attn_b200.inputs import DECODE, SEEDS, WINDOW, decode_inputs

pytestmark = pytest.mark.gpu


def paginate(k_cache, v_cache, seqlens, page_size, seed, share_first=False, junk_pages=None):
    """Scatter contiguous caches [B, Lmax, Hkv, D] into a shuffled page pool.

    Only the pages a sequence needs are mapped; the pool holds junk_pages
    unused pages besides (default: as many again), and they, every slot past
    a sequence's end and every page
    table entry past its last page are junk (NaN pages, entry -1), so a read of
    anything the call must not use shows up in the result.  With share_first,
    sequence 1 maps sequence 0's first page (prefix sharing)."""
    B, Lmax, Hkv, D = k_cache.shape
    max_pages = (Lmax + page_size - 1) // page_size
    need = [(int(seqlens[b]) + page_size - 1) // page_size for b in range(B)]
    num_pages = sum(need) + (sum(need) if junk_pages is None else junk_pages) + 1
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)
    kp = torch.full((num_pages, page_size, Hkv, D), float("nan"), dtype=k_cache.dtype)
    vp = torch.full((num_pages, page_size, Hkv, D), float("nan"), dtype=v_cache.dtype)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        L = int(seqlens[b])
        for lp in range(need[b]):
            phys = int(perm[nxt])
            nxt += 1
            table[b, lp] = phys
            t0, t1 = lp * page_size, min(L, (lp + 1) * page_size)
            kp[phys, :t1 - t0] = k_cache[b, t0:t1]
            vp[phys, :t1 - t0] = v_cache[b, t0:t1]
    if share_first and B > 1 and int(seqlens[1]) >= page_size and int(seqlens[0]) >= page_size:
        table[1, 0] = table[0, 0]
    return kp, vp, table


def run_paged(d, kp, vp, table, window, scale, num_splits=0):
    dev = "cuda"
    q = d["q"].to(dev)
    sl, s = d["seqlens"].to(dev), d["sinks"].to(dev)
    B, Hq, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, device=dev, dtype=torch.float32)
    nbytes = attn_sink_decode_paged_workspace_size(B, Hq, D, table.shape[1], kp.shape[1], window, num_splits)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    attn_sink_decode_paged(q, kp.to(dev), vp.to(dev), table.to(dev), sl, s, out, lse, window, scale, num_splits, ws)
    torch.cuda.synchronize()
    return out, lse


def run_contiguous(d, window, scale, num_splits=0):
    dev = "cuda"
    q = d["q"].to(dev)
    B, Hq, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, device=dev, dtype=torch.float32)
    nbytes = attn_sink_decode_workspace_size(B, Hq, D, d["k_cache"].shape[1], window, num_splits)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    attn_sink_decode(q, d["k_cache"].to(dev), d["v_cache"].to(dev), d["seqlens"].to(dev), d["sinks"].to(dev), out,
                     lse, window, scale, num_splits, ws)
    torch.cuda.synchronize()
    return out, lse


def oracle_per_sequence(d, window, scale):
    outs, lses = [], []
    for b in range(d["q"].shape[0]):
        L = int(d["seqlens"][b])
        o, l = oracle.decode(d["q"][b:b + 1], d["k_cache"][b:b + 1, :L], d["v_cache"][b:b + 1, :L],
                             d["seqlens"][b:b + 1], d["sinks"], window, scale)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs), np.concatenate(lses)


def small_inputs(seed=SEEDS["decode"] + 100):
    # ragged lengths that hit 1, page and tile boundaries and Lmax
    d = decode_inputs(8, 1000, 16, 2, 64, 1, 1000, torch.bfloat16, 0.5, 1.0, seed=seed)
    d["seqlens"] = torch.tensor([1, 7, 64, 65, 128, 333, 999, 1000], dtype=torch.int32)
    return d


_small_cache = {}


def _small():
    if "d" not in _small_cache:
        _small_cache["d"] = small_inputs()
    return _small_cache["d"]


@pytest.mark.parametrize("window", [0, 3, 64, WINDOW])
@pytest.mark.parametrize("page_size", [8, 16, 32, 64, 128])
def test_paged_matches_oracle(page_size, window):
    d = _small()
    scale = 1.0 / math.sqrt(64)
    kp, vp, table = paginate(d["k_cache"], d["v_cache"], d["seqlens"], page_size, seed=page_size + window)
    ref_o, ref_l = oracle_per_sequence(d, window, scale)
    for splits in (0, 1, 4):
        out, lse = run_paged(d, kp, vp, table, window, scale, splits)
        assert torch.isfinite(out.float()).all(), (page_size, window, splits)
        assert_close_bf16(out.float().cpu().numpy(), ref_o)
        assert_lse(lse.cpu().numpy(), ref_l)


@pytest.mark.parametrize("page_size", [16, 64])
def test_paged_equals_contiguous_dense(page_size):
    # dense: both calls start the split range at key 0, so the tiles (and the
    # arithmetic) are the same and the results agree bit for bit
    d = _small()
    scale = 0.125
    kp, vp, table = paginate(d["k_cache"], d["v_cache"], d["seqlens"], page_size, seed=7)
    for splits in (0, 2, 8):
        po, pl = run_paged(d, kp, vp, table, 0, scale, splits)
        co, cl = run_contiguous(d, 0, scale, splits)
        assert torch.equal(po, co), splits
        assert torch.equal(pl, cl), splits


def test_paged_shared_prefix_pages():
    d = _small()
    # sequence 1 re-uses sequence 0's first page: give it the same first keys
    d = {k: v.clone() for k, v in d.items()}
    d["seqlens"][0] = 200
    d["seqlens"][1] = 150
    d["k_cache"][1, :16] = d["k_cache"][0, :16]
    d["v_cache"][1, :16] = d["v_cache"][0, :16]
    kp, vp, table = paginate(d["k_cache"], d["v_cache"], d["seqlens"], 16, seed=3, share_first=True)
    assert table[1, 0] == table[0, 0]
    ref_o, ref_l = oracle_per_sequence(d, 0, 0.125)
    out, lse = run_paged(d, kp, vp, table, 0, 0.125)
    assert_close_bf16(out.float().cpu().numpy(), ref_o)
    assert_lse(lse.cpu().numpy(), ref_l)


_full = {}


def _full_inputs():
    if "d" not in _full:
        w = DECODE
        _full["d"] = decode_inputs(w.B, w.Lmax, w.Hq, w.Hkv, w.D, w.len_lo, w.len_hi, w.dtype, w.qkv_std, w.sink_std,
                                   seed=SEEDS["decode"])
    return _full["d"]


def test_paged_full_workload_dense_equals_contiguous():
    # the 64-sequence decode workload (Lmax 32768) in pages of 16 keys
    d = _full_inputs()
    scale = 1.0 / math.sqrt(64)
    kp, vp, table = paginate(d["k_cache"], d["v_cache"], d["seqlens"], 16, seed=11, junk_pages=256)
    po, pl = run_paged(d, kp, vp, table, 0, scale)
    co, cl = run_contiguous(d, 0, scale)
    assert torch.equal(po, co)
    assert torch.equal(pl, cl)


def test_paged_full_workload_banded_oracle():
    d = _full_inputs()
    scale = 1.0 / math.sqrt(64)
    kp, vp, table = paginate(d["k_cache"], d["v_cache"], d["seqlens"], 16, seed=12, junk_pages=256)
    out, lse = run_paged(d, kp, vp, table, WINDOW, scale)
    ref_o, ref_l = oracle_per_sequence(d, WINDOW, scale)
    assert_close_bf16(out.float().cpu().numpy(), ref_o)
    assert_lse(lse.cpu().numpy(), ref_l)
