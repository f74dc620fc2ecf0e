"""Shared helpers for the parity tests: tolerances and comparisons (no attention arithmetic)."""
import math

import numpy as np
import torch

# Parity tolerances: the exact fp32 path to 1e-5 max-abs; the bf16 path to
# 2e-2 max-abs and 5e-3 relative L2 (bf16 rounding of P before the PV product
# and of the stored output, against an fp64 reference).
FP32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
# LSE is computed in fp32 from exact products of bf16 inputs; its error is
# rounding of fp32 sums of O(L) terms, far below this bound.
LSE_MAX_ABS = 1e-3


def to_np(t):
    return t.detach().float().cpu().double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t, dtype=np.float64)


def errors(got, ref):
    g, r = to_np(got), to_np(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), "non-finite pattern differs"
    d = np.abs(g[fin] - r[fin])
    max_abs = float(d.max()) if d.size else 0.0
    den = float(np.sqrt((r[fin] ** 2).sum()))
    rel = float(np.sqrt((d ** 2).sum()) / den) if den > 0 else float(np.sqrt((d ** 2).sum()))
    return max_abs, rel


def assert_close_bf16(got, ref, what="", max_abs=BF16_MAX_ABS, rel_l2=BF16_REL_L2):
    ma, rl = errors(got, ref)
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max_abs={ma:.3e} rel_l2={rl:.3e}"
    return ma, rl


def assert_close_fp32(got, ref, what="", max_abs=FP32_MAX_ABS):
    ma, rl = errors(got, ref)
    assert ma <= max_abs, f"{what}: max_abs={ma:.3e}"
    return ma, rl


def assert_lse(got, ref, what="", max_abs=LSE_MAX_ABS):
    ma, _ = errors(got, ref)
    assert ma <= max_abs, f"{what}: lse max_abs={ma:.3e}"
    return ma
