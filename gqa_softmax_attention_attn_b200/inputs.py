"""Seeded synthetic inputs shared by the oracle tests, the CUDA parity tests and bench.py.

This module holds no attention arithmetic: it only draws random tensors on the
CPU with a torch ``Generator`` (seed = 1000 + workload number unless given),
in the fixed draw order q, k, v, sinks, dO, lengths, and casts them to the
compute dtype once.  The workloads are the five shapes of the gpt-oss attention
layer the pages describe (grouped-query heads 64/8, head dim 64, dense causal
and window-128 banded layers, contexts up to 128K).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    L: int
    Hq: int
    Hkv: int
    D: int
    dtype: torch.dtype
    qkv_std: float
    sink_std: float
    dout_std: float


@dataclass(frozen=True)
class Decode:
    name: str
    B: int
    Lmax: int
    len_lo: int
    len_hi: int
    Hq: int
    Hkv: int
    D: int
    dtype: torch.dtype
    qkv_std: float
    sink_std: float


# The five workloads (numbered 1..5); each prefill one is run dense and banded (window 128).
TINY_FP32 = Prefill("tiny-fp32 B1 L256 Hq8 Hkv2 D64", 1, 256, 8, 2, 64, torch.float32, 1.0, 1.0, 1.0)
PREFILL_20B = Prefill("gpt-oss-20b prefill B1 L4096 Hq64 Hkv8 D64 bf16", 1, 4096, 64, 8, 64, torch.bfloat16, 0.5, 1.0, 0.1)
TRAIN = Prefill("train fwd+bwd B8 L8192 Hq64 Hkv8 D64 bf16", 8, 8192, 64, 8, 64, torch.bfloat16, 0.5, 1.0, 0.1)
DECODE = Decode("decode B64 Lmax32768 len~U[1024,32768] Hq64 Hkv8 D64 bf16", 64, 32768, 1024, 32768, 64, 8, 64,
                torch.bfloat16, 0.5, 1.0)
LONG_BANDED = Prefill("long banded B1 L131072 Hq64 Hkv8 D64 bf16", 1, 131072, 64, 8, 64, torch.bfloat16, 0.5, 2.0, 0.1)
LONG_DENSE = Prefill("long dense B1 L32768 Hq64 Hkv8 D64 bf16", 1, 32768, 64, 8, 64, torch.bfloat16, 0.5, 2.0, 0.1)
WINDOW = 128

SEEDS = {"tiny": 1001, "prefill": 1002, "train": 1003, "decode": 1004, "long": 1005}


def prefill_inputs(B, Lq, Lk, Hq, Hkv, D, dtype=torch.bfloat16, qkv_std=0.5, sink_std=1.0,
                   dout_std=0.1, seed=0, with_dout=False, sink_fill=None):
    """Returns a dict of CPU tensors: q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D] in `dtype`,
    sinks [Hq] fp32, and (optionally) dout [B,Lq,Hq,D] in `dtype`."""
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Lq, Hq, D, generator=g) * qkv_std).to(dtype)
    k = (torch.randn(B, Lk, Hkv, D, generator=g) * qkv_std).to(dtype)
    v = (torch.randn(B, Lk, Hkv, D, generator=g) * qkv_std).to(dtype)
    sinks = torch.randn(Hq, generator=g) * sink_std
    if sink_fill is not None:
        sinks = torch.full((Hq,), float(sink_fill))
    out = {"q": q, "k": k, "v": v, "sinks": sinks.float()}
    if with_dout:
        out["dout"] = (torch.randn(B, Lq, Hq, D, generator=g) * dout_std).to(dtype)
    return out


def workload_inputs(w: Prefill, seed: int, with_dout=False):
    return prefill_inputs(w.B, w.L, w.L, w.Hq, w.Hkv, w.D, w.dtype, w.qkv_std, w.sink_std,
                          w.dout_std, seed=seed, with_dout=with_dout)


def decode_inputs(B, Lmax, Hq, Hkv, D, len_lo, len_hi, dtype=torch.bfloat16, qkv_std=0.5,
                  sink_std=1.0, seed=0):
    """q [B,Hq,D], k/v caches [B,Lmax,Hkv,D], seqlens [B] int32 ~ U{len_lo..len_hi}, sinks [Hq]."""
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Hq, D, generator=g) * qkv_std).to(dtype)
    k = (torch.randn(B, Lmax, Hkv, D, generator=g) * qkv_std).to(dtype)
    v = (torch.randn(B, Lmax, Hkv, D, generator=g) * qkv_std).to(dtype)
    sinks = (torch.randn(Hq, generator=g) * sink_std).float()
    lens = torch.randint(len_lo, len_hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    return {"q": q, "k_cache": k, "v_cache": v, "seqlens": lens, "sinks": sinks}


def sample_rows(B, Hq, Lq, n, seed, window=0, sinks=None):
    """Seeded (b, h, i) sample, stratified: a third among the first 128 rows
    (partial band), a third in the last 1% of rows, the rest uniform; when
    `sinks` is given, half of the uniform share is drawn from heads whose sink
    exceeds two standard deviations (strongly dominant sinks)."""
    g = torch.Generator().manual_seed(seed)
    n1 = n // 3
    n2 = n // 3
    n3 = n - n1 - n2
    b = torch.randint(0, B, (n,), generator=g)
    h = torch.randint(0, Hq, (n,), generator=g)
    i1 = torch.randint(0, min(128, Lq), (n1,), generator=g)
    tail = max(1, Lq // 100)
    i2 = torch.randint(Lq - tail, Lq, (n2,), generator=g)
    i3 = torch.randint(0, Lq, (n3,), generator=g)
    i = torch.cat([i1, i2, i3])
    if sinks is not None:
        s = sinks.float()
        strong = torch.nonzero(s > 2.0 * s.std()).flatten()
        if len(strong) > 0:
            k = n3 // 2
            pick = strong[torch.randint(0, len(strong), (k,), generator=g)]
            h[n1 + n2:n1 + n2 + k] = pick
    return b.int(), h.int(), i.int()


def quantize_e4m3_per_head(x):
    """A KV cache [B, L, Hkv, D] in FP8 e4m3 with one fp32 scale per KV head:
    scale_g = max|x[..., g, :]| / 448 (448 is the largest e4m3 value), codes =
    x / scale_g rounded to e4m3 by torch's cast.  Returns (codes as uint8, the
    one-byte storage of the cache; scales [Hkv] fp32).  This only prepares
    the input format; the attention arithmetic lives elsewhere."""
    xf = x.float()
    amax = xf.abs().amax(dim=(0, 1, 3)).clamp_min(1e-12)
    scales = (amax / 448.0).float()
    codes = (xf / scales[None, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scales.contiguous()
