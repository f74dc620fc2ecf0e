"""The FMA-pipe exp2 used by the forward kernel (fast_exp2x2: range reduction
plus a degree-3 minimax polynomial fitted by exp2_poly.py) against CUDA's own
exp2f, over the range the softmax feeds it."""
import ctypes
import os

import numpy as np
import pytest
import torch

from gqa_softmax_attention_attn_b200 import build

pytestmark = pytest.mark.gpu


def test_fast_exp2_relative_error_bound():
    lib = ctypes.CDLL(build.SELFTEST_LIB)
    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 20), torch.linspace(-1.0, 1.0, 1 << 16),
                   torch.tensor([0.0, -0.5, 0.5, -125.5, 7.999])]).float()
    if x.numel() % 2:
        x = torch.cat([x, torch.zeros(1)])
    xd = x.cuda()
    fast, mufu, ref = (torch.empty_like(xd) for _ in range(3))
    rc = lib.attn_sink_selftest_exp2(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(fast.data_ptr()),
                                     ctypes.c_void_p(mufu.data_ptr()), ctypes.c_void_p(ref.data_ptr()),
                                     ctypes.c_int(xd.numel()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    f, r = fast.double().cpu(), ref.double().cpu()
    ok = r > 1e-37  # normal range of the result
    rel = ((f - r).abs() / r)[ok]
    assert rel.max().item() < 1.0e-4, rel.max().item()  # polynomial bound 7.5e-5 + fp32 rounding
    assert torch.isfinite(f).all() and (f >= 0).all()
    # results below 1e-37 (x < -122.9, and the clamp at x = -126) stay tiny and non-negative
    assert (f[~ok] <= 1.001e-37).all()


def test_pipe_rate_microbenchmarks():
    # measured results per clock per SM of MUFU ex2 and of the bf16x2 pack;
    # the rates bench.py turns into the exponential roof
    lib = ctypes.CDLL(build.SELFTEST_LIB)
    lib.attn_sink_selftest_pipe_rate.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double)]
    rates = []
    for which in (0, 1):
        r = ctypes.c_double(0.0)
        assert lib.attn_sink_selftest_pipe_rate(which, ctypes.byref(r)) == 0
        rates.append(r.value)
    assert 4.0 <= rates[0] <= 128.0, rates
    assert 4.0 <= rates[1] <= 256.0, rates
    r = ctypes.c_double(0.0)
    assert lib.attn_sink_selftest_pipe_rate(7, ctypes.byref(r)) == -1
