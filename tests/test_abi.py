"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments on the host before touching any device (CPU only)."""
import ctypes
import os
import re

import pytest

import gqa_softmax_attention_attn_b200 as attn
from gqa_softmax_attention_attn_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_sink.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, ARCH, WORKSPACE, CUDA, TIMEOUT, NODEV = 0, -1, -2, -3, -4, -5, -6, -7, -8


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"ATTN_SINK_API\s+[\w\s\*]+?\b(attn_sink_\w+)\s*\(", txt)))


def test_header_declares_the_three_calls():
    syms = declared_symbols()
    for s in ("attn_sink_fwd", "attn_sink_decode", "attn_sink_bwd"):
        assert s in syms


def test_library_exports_every_declared_symbol():
    lib = attn.load()
    for s in declared_symbols():
        assert hasattr(lib, s), s
    out = os.popen(f"nm -D --defined-only {_native.LIB_PATH}").read()
    exported = set(re.findall(r" T (\w+)", out))
    assert set(declared_symbols()) <= exported
    # nothing else leaks out of the library
    assert all(e.startswith("attn_sink_") for e in exported), exported


def test_strerror_and_version():
    assert attn.attn_sink_version() >= 100
    for code in (OK, INVALID, UNSUPPORTED, MISALIGNED, ARCH, WORKSPACE, CUDA, TIMEOUT, NODEV):
        assert len(attn.strerror(code)) > 0
    assert attn.strerror(-99) == "unknown status"


def _fake(n=8):
    # distinct, 256-byte aligned, non-null addresses; never dereferenced by the host checks
    return [0x7f0000000000 + 0x1000 * i for i in range(n)]


def test_fwd_host_checks():
    lib = attn.load()
    q, k, v, s, o, l = _fake(6)
    assert lib.attn_sink_fwd(None, k, v, s, o, l, 1, 16, 16, 8, 2, 64, 0, 0.125, 1, None) == INVALID
    assert lib.attn_sink_fwd(q, k, v, s, o, l, 0, 16, 16, 8, 2, 64, 0, 0.125, 1, None) == INVALID
    assert lib.attn_sink_fwd(q, k, v, s, o, l, 1, 16, 16, 8, 3, 64, 0, 0.125, 1, None) == INVALID
    assert lib.attn_sink_fwd(q, k, v, s, o, l, 1, 16, 16, 8, 2, 128, 0, 0.125, 1, None) == UNSUPPORTED
    assert lib.attn_sink_fwd(q, k, v, s, o, l, 1, 16, 16, 8, 2, 64, 0, 0.125, 7, None) == UNSUPPORTED
    assert lib.attn_sink_fwd(q + 2, k, v, s, o, l, 1, 16, 16, 8, 2, 64, 0, 0.125, 1, None) == MISALIGNED
    # bf16: the scale must be positive and finite
    for bad in (0.0, -0.125, float("inf"), float("nan")):
        assert lib.attn_sink_fwd(q, k, v, s, o, l, 1, 16, 16, 8, 2, 64, 0, bad, 1, None) == UNSUPPORTED, bad


def test_decode_host_checks():
    lib = attn.load()
    q, kc, vc, sl, s, o, l, ws = _fake(8)
    args = [q, kc, vc, sl, s, o, l, 4, 4096, 8, 2, 64, 0, 0.125]
    assert lib.attn_sink_decode(*args, 33, ws, 1 << 20, 1, None) == INVALID
    need = attn.attn_sink_decode_workspace_size(4, 8, 64, 4096, 0, 8)
    assert need == 4 * 8 * 8 * (64 + 2) * 4
    assert lib.attn_sink_decode(*args, 8, None, 0, 1, None) == WORKSPACE
    assert lib.attn_sink_decode(*args, 8, ws, need - 4, 1, None) == WORKSPACE
    # one split needs no workspace
    assert attn.attn_sink_decode_workspace_size(4, 8, 64, 4096, 128, 0) == 0


def test_fwd_varlen_host_checks():
    lib = attn.load()
    q, k, v, s, o, l, cq, ck = _fake(8)

    def call(cu_q=cq, cu_k=ck, B=3, max_q=100, total_q=200, total_k=200, Hq=8, Hkv=2, D=64, scale=0.125):
        return lib.attn_sink_fwd_varlen(q, k, v, s, o, l, cu_q, cu_k, B, max_q, total_q, total_k, Hq, Hkv, D, 0,
                                        scale, None)

    assert call(cu_q=None) == INVALID
    assert call(cu_k=None) == INVALID
    assert call(B=0) == INVALID
    assert call(max_q=0) == INVALID
    assert call(total_q=0) == INVALID
    assert call(total_k=0) == INVALID
    assert call(Hkv=3) == INVALID
    assert call(D=128) == UNSUPPORTED
    assert call(scale=0.0) == UNSUPPORTED
    assert call(cu_q=cq + 4) == MISALIGNED


def test_decode_fp8_host_checks():
    lib = attn.load()
    q, kc, vc, ks, vs, sl, s, o = _fake(8)
    l, ws = _fake(10)[8:]

    def call(k_scale=ks, v_scale=vs, B=4, Lmax=4096, Hq=8, Hkv=2, D=64, splits=8, w=ws, wbytes=1 << 20):
        return lib.attn_sink_decode_fp8(q, kc, vc, k_scale, v_scale, sl, s, o, l, B, Lmax, Hq, Hkv, D, 0, 0.125,
                                        splits, w, wbytes, None)

    assert call(k_scale=None) == INVALID
    assert call(v_scale=None) == INVALID
    assert call(splits=33) == INVALID
    assert call(Hkv=3) == INVALID
    assert call(D=128) == UNSUPPORTED
    assert call(k_scale=ks + 4) == MISALIGNED
    assert call(w=None, wbytes=0) == WORKSPACE
    need = attn.attn_sink_decode_workspace_size(4, 8, 64, 4096, 0, 8)
    assert call(wbytes=need - 4) == WORKSPACE


def test_fwd_fp8_host_checks():
    """Argument checks of the FP8 prefill, all on the host (no kernel runs)."""
    lib = attn.load()
    q, k, v, qs, ks, vs, s, o = _fake(8)
    l = _fake(9)[8]

    ws = _fake(10)[9]
    need = attn.attn_sink_fwd_fp8_workspace_size(1, 128, 2, 64)
    assert need == 1 * 128 * 2 * 64 * 2

    def call(q_scale=qs, k_scale=ks, B=1, Lq=128, Lk=128, Hq=8, Hkv=2, D=64, scale=0.125, qq=q, w=ws, wbytes=need):
        return lib.attn_sink_fwd_fp8(qq, k, v, q_scale, k_scale, vs, s, o, l, B, Lq, Lk, Hq, Hkv, D, 0, scale, w,
                                     wbytes, None)

    assert call(q_scale=None) == INVALID
    assert call(k_scale=None) == INVALID
    assert call(B=0) == INVALID
    assert call(Hkv=3) == INVALID
    assert call(D=128) == UNSUPPORTED
    assert call(scale=0.0) == UNSUPPORTED
    assert call(scale=-1.0) == UNSUPPORTED
    assert call(qq=q + 4) == MISALIGNED
    assert call(q_scale=qs + 4) == MISALIGNED
    assert call(w=None, wbytes=0) == WORKSPACE
    assert call(wbytes=need - 1) == WORKSPACE
    assert call(w=ws + 4) == MISALIGNED


def test_fwd_host_buffers_checks():
    """Argument checks of the host-buffer prefill, all on the host (nothing is enqueued)."""
    lib = attn.load()
    q, k, v, s, o, l, ws = _fake(7)
    need = attn.attn_sink_fwd_host_workspace_size(2, 100, 120, 8, 2, 64)
    # q and out, k and v, lse [B, Hq, Lq], sinks; 256-byte sections
    a256 = lambda x: (x + 255) // 256 * 256
    assert need == (2 * a256(2 * 100 * 8 * 64 * 2) + 2 * a256(2 * 120 * 2 * 64 * 2) + a256(2 * 8 * 100 * 4) + a256(8 * 4))
    assert attn.attn_sink_fwd_host_workspace_size(2, 100, 120, 8, 3, 64) == 0

    def call(B=2, Lq=100, Lk=120, Hq=8, Hkv=2, D=64, scale=0.125, chunks=4, qq=q, w=ws, wbytes=need):
        return lib.attn_sink_fwd_host(qq, k, v, s, o, l, B, Lq, Lk, Hq, Hkv, D, 0, scale, chunks, w, wbytes, None)

    assert call(qq=None) == INVALID
    assert call(chunks=0) == INVALID
    assert call(chunks=65) == INVALID
    assert call(B=0) == INVALID
    assert call(Hkv=3) == INVALID
    assert call(D=128) == UNSUPPORTED
    assert call(scale=0.0) == UNSUPPORTED
    assert call(Lq=121) == UNSUPPORTED  # more queries than keys
    assert call(w=None, wbytes=0) == WORKSPACE
    assert call(wbytes=need - 1) == WORKSPACE
    assert call(w=ws + 4) == MISALIGNED


def test_decode_paged_host_checks():
    lib = attn.load()
    q, kp, vp, pt, sl, s, o, l = _fake(8)
    ws = _fake(9)[8]

    def call(B=4, max_pages=256, page_size=16, num_pages=1024, Hq=8, Hkv=2, D=64, window=0, splits=0,
             w=ws, wbytes=1 << 20, dtype=1, ptab=pt):
        return lib.attn_sink_decode_paged(q, kp, vp, ptab, sl, s, o, l, B, max_pages, page_size, num_pages, Hq, Hkv,
                                          D, window, 0.125, splits, w, wbytes, dtype, None)

    for bad_ps in (0, -16, 4, 12, 24, 48, 100):
        assert call(page_size=bad_ps) == INVALID, bad_ps
    assert call(max_pages=0) == INVALID
    assert call(num_pages=0) == INVALID
    assert call(max_pages=1 << 25, page_size=64) == INVALID  # 2^31 keys per sequence
    assert call(splits=33) == INVALID
    assert call(ptab=None) == INVALID
    assert call(dtype=0) == UNSUPPORTED  # bf16 only
    assert call(D=128) == UNSUPPORTED
    assert call(ptab=pt + 4) == MISALIGNED
    # dense, 8 splits over 256 pages of 16 keys: chunk 512, 8 partials per (b, h)
    need = attn.attn_sink_decode_paged_workspace_size(4, 8, 64, 256, 16, 0, 8)
    assert need == 4 * 8 * 8 * (64 + 2) * 4
    assert call(splits=8, w=None, wbytes=0) == WORKSPACE
    assert call(splits=8, wbytes=need - 4) == WORKSPACE
    # banded: the split range may start up to 63 keys early (64-key aligned tiles)
    assert attn.attn_sink_decode_paged_workspace_size(4, 8, 64, 256, 16, 128, 0) == 0
    # 4 splits asked over 191 keys: 64-key chunks, so 3 partials
    assert attn.attn_sink_decode_paged_workspace_size(4, 8, 64, 256, 16, 128, 4) == 4 * 8 * 3 * 66 * 4
    assert attn.attn_sink_decode_paged_workspace_size(4, 8, 64, 256, 12, 0, 8) == 0  # invalid page size


def test_bwd_host_checks():
    lib = attn.load()
    p = _fake(12)
    need = attn.attn_sink_bwd_workspace_size(2, 32, 32, 8, 2, 64, 1)
    assert need > 0
    base = p[:11] + [2, 32, 32, 8, 2, 64, 0, 0.125]
    assert lib.attn_sink_bwd(*base, None, 0, 1, None) == WORKSPACE
    assert lib.attn_sink_bwd(*base, p[11], need - 1, 1, None) == WORKSPACE
    bad = [None] + p[1:11] + [2, 32, 32, 8, 2, 64, 0, 0.125]
    assert lib.attn_sink_bwd(*bad, p[11], need, 1, None) == INVALID


def test_no_device_is_reported_cleanly():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a device is present")
    lib = attn.load()
    q, k, v, s, o, l = _fake(6)
    assert lib.attn_sink_fwd(q, k, v, s, o, l, 1, 16, 16, 8, 2, 64, 0, 0.125, 1, None) == NODEV
    assert lib.attn_sink_get_device_status(None) == NODEV


def test_wait_timeout_setting_round_trips():
    old = attn.attn_sink_set_wait_timeout_ns(123456789)
    assert attn.attn_sink_set_wait_timeout_ns(old) == 123456789


def test_qkv_prologue_host_checks():
    lib = attn.load()
    qkv, b, pos, rows, q, k, v = _fake(7)

    def call(qkv_=qkv, pos_=pos, rows_=rows, T=10, Hq=8, Hkv=2, D=64, nrows=10, theta=10000.0, factor=32.0, L0=4096,
             bf=32.0, bs=1.0, inter=0):
        return lib.attn_sink_qkv_prologue(qkv_, b, pos_, rows_, q, k, v, T, Hq, Hkv, D, nrows, theta, factor, L0, bf,
                                          bs, inter, None)

    assert call(qkv_=None) == INVALID
    assert call(pos_=None) == INVALID
    assert call(T=0) == INVALID
    assert call(Hkv=3) == INVALID
    assert call(D=128) == UNSUPPORTED
    assert call(rows_=None, nrows=5) == INVALID  # row t must exist without a row map
    assert call(theta=1.0) == INVALID
    assert call(factor=0.0) == INVALID
    assert call(L0=0) == INVALID  # YaRN needs the original context
    assert call(bf=1.0, bs=1.0) == INVALID
    assert call(inter=2) == INVALID
    assert call(pos_=pos + 4) == MISALIGNED
