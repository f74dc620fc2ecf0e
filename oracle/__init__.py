"""fp64 CPU oracle for sink-softmax GQA attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
product path (``gqa_softmax_attention_attn_b200``) never imports it, and the
two share no code.

The arithmetic lives in ``attn_sink_oracle.c`` (plain C, fp64, OpenMP); this
module only compiles it with gcc and marshals numpy float64 arrays.  The
definition it follows is stated in the C file's header ("GPT-OSS on day 0",
sections "Attention: GQA with Attention Sinks" and "Sink Attention").

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against library routines (PyTorch CPU fp64 SDPA and autograd, torch's FP8
widening), closed forms, invariants, brute force and finite differences.  The pages print no worked
example, so no stored golden values from the pages exist.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_sink_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/_build/liboracle.so (generic x86-64 flags)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load(path: str | None = None):
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(path or build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        Dd = ctypes.c_double
        lib.oracle_fwd.argtypes = [P] * 6 + [I] * 7 + [Dd]
        lib.oracle_fwd_rows.argtypes = [P] * 7 + [I] + [P, P] + [I] * 7 + [Dd]
        lib.oracle_decode.argtypes = [P] * 7 + [I] * 6 + [Dd]
        lib.oracle_bwd.argtypes = [P] * 9 + [I] * 7 + [Dd]
        lib.oracle_row_stats.argtypes = [P] * 7 + [I] * 7 + [Dd]
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


class use_library:
    """Context manager that points this module at another build of the C
    oracle (used only by the mutation test, which compiles planted mistakes)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = None
        _load(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def fwd(q, k, v, sinks, window: int, scale: float):
    """q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D], sinks [Hq] -> (out [B,Lq,Hq,D], lse [B,Hq,Lq])."""
    q, k, v, sinks = _f64(q), _f64(k), _f64(v), _f64(sinks)
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    assert Hq % Hkv == 0 and sinks.shape == (Hq,)
    out = np.empty_like(q)
    lse = np.empty((B, Hq, Lq))
    _load().oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(out), _ptr(lse),
                       B, Lq, Lk, Hq, Hkv, D, int(window), float(scale))
    return out, lse


def fwd_rows(q, k, v, sinks, rows_b, rows_h, rows_i, window: int, scale: float):
    """Forward for sampled rows only: returns (out_rows [n,D], lse_rows [n])."""
    q, k, v, sinks = _f64(q), _f64(k), _f64(v), _f64(sinks)
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    rb = np.ascontiguousarray(rows_b, dtype=np.int32)
    rh = np.ascontiguousarray(rows_h, dtype=np.int32)
    ri = np.ascontiguousarray(rows_i, dtype=np.int32)
    n = len(rb)
    out = np.empty((n, D))
    lse = np.empty((n,))
    _load().oracle_fwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(rb), _ptr(rh), _ptr(ri), n,
                            _ptr(out), _ptr(lse), B, Lq, Lk, Hq, Hkv, D, int(window), float(scale))
    return out, lse


def decode(q, k_cache, v_cache, seqlens, sinks, window: int, scale: float):
    """q [B,Hq,D], caches [B,Lmax,Hkv,D], seqlens [B] -> (out [B,Hq,D], lse [B,Hq])."""
    q, kc, vc, sinks = _f64(q), _f64(k_cache), _f64(v_cache), _f64(sinks)
    sl = np.ascontiguousarray(np.asarray(seqlens.cpu() if hasattr(seqlens, "cpu") else seqlens), dtype=np.int32)
    B, Hq, D = q.shape
    Lmax, Hkv = kc.shape[1], kc.shape[2]
    assert sl.min() >= 1 and sl.max() <= Lmax
    out = np.empty_like(q)
    lse = np.empty((B, Hq))
    _load().oracle_decode(_ptr(q), _ptr(kc), _ptr(vc), _ptr(sl), _ptr(sinks), _ptr(out), _ptr(lse),
                          B, Lmax, Hq, Hkv, D, int(window), float(scale))
    return out, lse


def bwd(q, k, v, sinks, dout, window: int, scale: float):
    """Returns (dq, dk, dv, dsinks) in fp64, recomputing the forward internally."""
    q, k, v, sinks, dout = _f64(q), _f64(k), _f64(v), _f64(sinks), _f64(dout)
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    ds = np.empty((Hq,))
    _load().oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                       _ptr(ds), B, Lq, Lk, Hq, Hkv, D, int(window), float(scale))
    return dq, dk, dv, ds


def row_stats(q, k, v, sinks, dout, window: int, scale: float):
    """Per-row D_i = <dO_i, O_i> and P_sink_i = exp(sink - LSE_i), each [B,Hq,Lq]."""
    q, k, v, sinks, dout = _f64(q), _f64(k), _f64(v), _f64(sinks), _f64(dout)
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    Dr = np.empty((B, Hq, Lq))
    Ps = np.empty((B, Hq, Lq))
    _load().oracle_row_stats(_ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(dout), _ptr(Dr), _ptr(Ps),
                             B, Lq, Lk, Hq, Hkv, D, int(window), float(scale))
    return Dr, Ps


def _e4m3_from_fields(c):
    """fp64 values of FP8 E4M3 codes c (OCP 8-bit floating point, E4M3: 1 sign
    bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds
    the subnormals m * 2^-9; no infinities; codes 0x7f and 0xff are NaN),
    computed field by field from that definition."""
    c = np.asarray(c, dtype=np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.power(2.0, e.astype(np.float64) - 7.0)
    sub = m * 2.0 ** -9
    v = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & ((c & 7) == 7), np.nan, v)


_E4M3 = _e4m3_from_fields(np.arange(256))  # the definition, once per code


def e4m3_values(codes):
    """fp64 values of an array of E4M3 codes (uint8), by the definition above."""
    c = codes.detach().cpu().view(__import__("torch").uint8).numpy() if hasattr(codes, "detach") else codes
    return _E4M3[np.asarray(c, dtype=np.uint8)]


def decode_fp8(q, k_codes, v_codes, k_scale, v_scale, seqlens, sinks, window: int, scale: float):
    """Decode over an e4m3 KV cache: every code is widened to its exact value
    and multiplied by its KV head's scale in fp64, then the decode definition
    runs unchanged.  Caches [B, Lmax, Hkv, D] of codes; scales [Hkv]."""
    ks = np.asarray(_f64(k_scale))
    vs = np.asarray(_f64(v_scale))
    k = e4m3_values(k_codes) * ks[None, None, :, None]
    v = e4m3_values(v_codes) * vs[None, None, :, None]
    return decode(q, k, v, seqlens, sinks, window, scale)


def fwd_fp8(q_codes, k_codes, v_codes, q_scale, k_scale, v_scale, sinks, window: int, scale: float):
    """Prefill forward over e4m3 inputs: every code is widened to its exact
    value and multiplied by its head's scale in fp64 (q per query head, k and
    v per KV head), then the forward definition runs unchanged.  q [B, Lq,
    Hq, D], k/v [B, Lk, Hkv, D] codes; scales [Hq], [Hkv], [Hkv]."""
    qs = np.asarray(_f64(q_scale))
    ks = np.asarray(_f64(k_scale))
    vs = np.asarray(_f64(v_scale))
    q = e4m3_values(q_codes) * qs[None, None, :, None]
    k = e4m3_values(k_codes) * ks[None, None, :, None]
    v = e4m3_values(v_codes) * vs[None, None, :, None]
    return fwd(q, k, v, sinks, window, scale)


def fwd_varlen(q, k, v, sinks, cu_q, cu_k, window: int, scale: float):
    """Packed ragged sequences: sequence b is the independent problem
    q[cu_q[b]:cu_q[b+1]] against k, v[cu_k[b]:cu_k[b+1]], run through fwd with
    B = 1.  q [total_q, Hq, D], k/v [total_k, Hkv, D] -> (out [total_q, Hq, D],
    lse [Hq, total_q]); empty sequences contribute nothing."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = [int(x) for x in (cu_q.tolist() if hasattr(cu_q, "tolist") else cu_q)]
    ck = [int(x) for x in (cu_k.tolist() if hasattr(cu_k, "tolist") else cu_k)]
    total_q, Hq, D = q.shape
    out = np.zeros((total_q, Hq, D))
    lse = np.zeros((Hq, total_q))
    for b in range(len(cq) - 1):
        a, e = cq[b], cq[b + 1]
        if e <= a:
            continue
        o, l = fwd(q[None, a:e], k[None, ck[b]:ck[b + 1]], v[None, ck[b]:ck[b + 1]], sinks, window, scale)
        out[a:e] = o[0]
        lse[:, a:e] = l[0]
    return out, lse


def yarn_frequencies(D: int, base: float, factor: float = 1.0, original_max_pos: float = 0.0,
                     beta_fast: float = 32.0, beta_slow: float = 1.0):
    """Rotary frequencies of the D/2 pairs and the attention factor, in fp64.

    Plain rotary embedding: f_i = base^(-2i/D).  YaRN (factor > 1), in the
    DeepSeek-V3 form the pages point to ("GPT-OSS on day 0", section
    "Attention: GQA with Attention Sinks"): d(n) = D ln(L0 / (2 pi n)) /
    (2 ln base) is the pair index at which a full wavelength fits n times
    into the original context L0; between d(beta_fast) and d(beta_slow) a
    ramp linear in the pair index moves the frequency from f_i (kept) to
    f_i / factor (interpolated); the attention factor is 0.1 ln(factor) + 1."""
    i = np.arange(D // 2, dtype=np.float64)
    f = np.power(float(base), -2.0 * i / D)
    if not factor > 1.0:
        return f, 1.0
    d = lambda n: D * np.log(original_max_pos / (2.0 * np.pi * n)) / (2.0 * np.log(base))
    lo, hi = d(beta_fast), d(beta_slow)
    ramp = np.clip((i - lo) / (hi - lo), 0.0, 1.0) if hi > lo else (i >= lo).astype(np.float64)
    keep = 1.0 - ramp
    return f * keep + (f / factor) * (1.0 - keep), 0.1 * np.log(factor) + 1.0


def rotate(x, positions, freqs, attn_factor, interleaved=False):
    """Rotary embedding of x [T, H, D] (fp64): pair i of token t turns by the
    angle positions[t] * freqs[i], scaled by attn_factor.  Pairs are
    (i, i + D/2), or (2i, 2i + 1) when interleaved."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * freqs[None, :]
    c = (np.cos(ang) * attn_factor)[:, None, :]
    s = (np.sin(ang) * attn_factor)[:, None, :]
    a, b = (x[..., 0::2], x[..., 1::2]) if interleaved else (x[..., :D // 2], x[..., D // 2:])
    out = np.empty_like(x)
    ra, rb = a * c - b * s, b * c + a * s
    if interleaved:
        out[..., 0::2], out[..., 1::2] = ra, rb
    else:
        out[..., :D // 2], out[..., D // 2:] = ra, rb
    return out


def qkv_prologue(qkv, bias, positions, Hq: int, Hkv: int, D: int, base: float, factor: float = 1.0,
                 original_max_pos: float = 0.0, beta_fast: float = 32.0, beta_slow: float = 1.0,
                 interleaved: bool = False):
    """The step before attention: y = qkv + bias, split into q [T, Hq, D],
    k [T, Hkv, D], v [T, Hkv, D]; q and k rotated at their token's position.
    Returns (q, k, v) in fp64."""
    y = _f64(qkv)
    if bias is not None:
        y = y + _f64(bias)[None, :]
    T = y.shape[0]
    y = y.reshape(T, Hq + 2 * Hkv, D)
    pos = np.asarray(positions.cpu() if hasattr(positions, "cpu") else positions, dtype=np.float64)
    f, a = yarn_frequencies(D, base, factor, original_max_pos, beta_fast, beta_slow)
    q = rotate(y[:, :Hq], pos, f, a, interleaved)
    k = rotate(y[:, Hq:Hq + Hkv], pos, f, a, interleaved)
    return q, k, y[:, Hq + Hkv:].copy()
