"""Pins for the fp64 oracle, against things other than itself (CPU only).

The pages print no worked example, so the oracle is pinned by:
  * library routines: PyTorch CPU fp64 scaled_dot_product_attention (SDPA) and
    autograd through it -- sink = -inf must reduce to ordinary causal GQA
    attention ("GPT-OSS on day 0", section "Attention: GQA with Attention
    Sinks": the sink only adds a logit), and sink attention must equal SDPA
    over keys augmented with one zero-value key whose logit is the sink
    (section "Sink Attention": the sink is a bias term entering the softmax
    but carrying no value row);
  * closed forms: window = 1, window = 2, a dominant sink;
  * invariants: row mass + sink mass = 1, a common shift of all logits,
    window >= Lk equals dense bit for bit;
  * brute force on tiny inputs written as a separate pure-Python path;
  * central finite differences for the backward.
Masks in these tests are built with torch.tril(diagonal=...) (a library
routine), independently of the oracle's index arithmetic.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from gqa_softmax_attention_attn_b200.inputs import decode_inputs, prefill_inputs

TOL = 1e-11


def _mask_bool(Lq, Lk, window):
    """Visible[i, j] with bottom-right causal alignment, via torch.tril."""
    ones = torch.ones(Lq, Lk, dtype=torch.bool)
    vis = torch.tril(ones, diagonal=Lk - Lq)
    if window > 0:
        vis = vis & ~torch.tril(ones, diagonal=Lk - Lq - window)
    return vis


def _sdpa_aug(q, k, v, sinks, scale, window, grad=False):
    """Sink attention as SDPA over keys augmented with a zero key whose additive
    mask entry is the sink logit; an extra value channel that is 1 only on the
    sink key returns the sink's probability P_sink, hence LSE = sink - ln P_sink.
    q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D] (fp64)."""
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    qt = q.permute(0, 2, 1, 3)
    kt = k.permute(0, 2, 1, 3)
    vt = v.permute(0, 2, 1, 3)
    zk = torch.zeros(B, Hkv, 1, D, dtype=q.dtype)
    k_aug = torch.cat([kt, zk], dim=2)
    v_aug = torch.cat([vt, zk], dim=2)
    chan = torch.zeros(B, Hkv, Lk + 1, 1, dtype=q.dtype)
    chan[:, :, Lk, 0] = 1.0
    v_aug = torch.cat([v_aug, chan], dim=3)
    vis = _mask_bool(Lq, Lk, window)
    base = torch.zeros(Lq, Lk, dtype=q.dtype).masked_fill(~vis, float("-inf"))
    mask = torch.cat([base.expand(Hq, Lq, Lk),
                      sinks.view(Hq, 1, 1).expand(Hq, Lq, 1)], dim=2).unsqueeze(0)
    o = F.scaled_dot_product_attention(qt, k_aug, v_aug, attn_mask=mask, scale=scale, enable_gqa=True)
    o = o.permute(0, 2, 1, 3)
    out = o[..., :D]
    psink = o[..., D]  # [B, Lq, Hq]
    lse = sinks.view(1, 1, Hq) - torch.log(psink)
    return out, lse.permute(0, 2, 1)


def _inp(B, Lq, Lk, Hq, Hkv, D, seed, sink_std=1.0, with_dout=False, sink_fill=None):
    t = prefill_inputs(B, Lq, Lk, Hq, Hkv, D, dtype=torch.float64, qkv_std=1.0, sink_std=sink_std,
                       dout_std=1.0, seed=seed, with_dout=with_dout, sink_fill=sink_fill)
    t["sinks"] = t["sinks"].double()
    return t


@pytest.mark.parametrize("Lq,Lk", [(33, 33), (20, 47), (1, 9)])
def test_sink_neg_inf_is_plain_causal_gqa_sdpa(Lq, Lk):
    t = _inp(2, Lq, Lk, 8, 2, 16, seed=1, sink_fill=float("-inf"))
    scale = 0.3
    out, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, scale)
    vis = _mask_bool(Lq, Lk, 0)
    ref = F.scaled_dot_product_attention(t["q"].permute(0, 2, 1, 3), t["k"].permute(0, 2, 1, 3),
                                         t["v"].permute(0, 2, 1, 3), attn_mask=vis, scale=scale,
                                         enable_gqa=True).permute(0, 2, 1, 3)
    assert np.abs(out - ref.numpy()).max() < TOL
    if Lq == Lk:
        ref2 = F.scaled_dot_product_attention(t["q"].permute(0, 2, 1, 3), t["k"].permute(0, 2, 1, 3),
                                              t["v"].permute(0, 2, 1, 3), is_causal=True, scale=scale,
                                              enable_gqa=True).permute(0, 2, 1, 3)
        assert np.abs(out - ref2.numpy()).max() < TOL


@pytest.mark.parametrize("window", [0, 1, 5, 16])
@pytest.mark.parametrize("Lq,Lk,Hq,Hkv", [(40, 40, 8, 2), (17, 30, 4, 4), (25, 25, 6, 1)])
def test_matches_augmented_sdpa(window, Lq, Lk, Hq, Hkv):
    t = _inp(2, Lq, Lk, Hq, Hkv, 8, seed=2 + window)
    scale = 1.0 / math.sqrt(8)
    out, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, scale)
    ref_o, ref_lse = _sdpa_aug(t["q"], t["k"], t["v"], t["sinks"], scale, window)
    assert np.abs(out - ref_o.numpy()).max() < TOL
    assert np.abs(lse - ref_lse.numpy()).max() < 1e-10


def test_window_ge_lk_is_dense_bitwise():
    t = _inp(1, 50, 50, 4, 2, 16, seed=3)
    o0, l0 = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, 0.25)
    for w in (50, 51, 1000):
        o1, l1 = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], w, 0.25)
        assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def test_window_one_closed_form():
    """window = 1: each row sees only its own key, so O_i = v_i * sigmoid(z_ii - sink)."""
    t = _inp(1, 30, 30, 4, 2, 8, seed=4)
    scale = 0.4
    out, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 1, scale)
    q, k, v, s = t["q"].numpy(), t["k"].numpy(), t["v"].numpy(), t["sinks"].numpy()
    for h in range(4):
        g = h // 2
        z = scale * np.einsum("id,id->i", q[0, :, h], k[0, :, g])
        sig = 1.0 / (1.0 + np.exp(-(z - s[h])))
        assert np.abs(out[0, :, h] - v[0, :, g] * sig[:, None]).max() < 1e-12
        assert np.abs(lse[0, h] - np.logaddexp(z, s[h])).max() < 1e-12


def test_window_two_closed_form():
    t = _inp(1, 12, 12, 2, 1, 4, seed=5)
    scale = 0.7
    out, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 2, scale)
    q, k, v, s = t["q"].numpy(), t["k"].numpy(), t["v"].numpy(), t["sinks"].numpy()
    for h in range(2):
        for i in range(12):
            zs = [scale * q[0, i, h] @ k[0, j, 0] for j in range(max(0, i - 1), i + 1)]
            vs = [v[0, j, 0] for j in range(max(0, i - 1), i + 1)]
            den = math.exp(s[h]) + sum(math.exp(z) for z in zs)
            o = sum(math.exp(z) * vv for z, vv in zip(zs, vs)) / den
            assert np.abs(out[0, i, h] - o).max() < 1e-12
            assert abs(lse[0, h, i] - math.log(den)) < 1e-12


def test_dominant_sink_drives_output_to_zero():
    t = _inp(1, 40, 40, 4, 2, 16, seed=6, sink_fill=50.0)
    scale = 0.25
    out, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, scale)
    z = scale * torch.einsum("bihd,bjhd->bhij", t["q"], t["k"].repeat_interleave(2, dim=2))
    bound = math.exp(float(z.max()) - 50.0) * float(t["v"].abs().max()) * 40
    assert np.abs(out).max() <= bound
    assert np.abs(out).max() < 1e-12
    assert np.abs(lse - 50.0).max() < 1e-12


@pytest.mark.parametrize("window", [0, 7])
def test_row_mass_plus_sink_mass_is_one(window):
    t = _inp(2, 31, 31, 8, 2, 16, seed=7)
    scale = 0.25
    _, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, scale)
    z = scale * torch.einsum("bihd,bjhd->bhij", t["q"], t["k"].repeat_interleave(4, dim=2))
    vis = _mask_bool(31, 31, window)
    lse_t = torch.from_numpy(lse)
    mass = (torch.exp(z - lse_t[..., None]) * vis).sum(-1) + torch.exp(t["sinks"].view(1, 8, 1) - lse_t)
    assert (mass - 1.0).abs().max() < 1e-12


def test_common_logit_shift_invariance():
    """Appending a coordinate c/scale to every q and 1 to every k adds c to all
    z_ij; adding c to the sink too must leave O unchanged and shift LSE by c."""
    t = _inp(1, 20, 20, 4, 2, 8, seed=8)
    scale, c = 0.5, 3.7
    o0, l0 = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, scale)
    q1 = torch.cat([t["q"], torch.full((1, 20, 4, 1), c / scale, dtype=torch.float64)], -1)
    k1 = torch.cat([t["k"], torch.ones(1, 20, 2, 1, dtype=torch.float64)], -1)
    v1 = torch.cat([t["v"], torch.zeros(1, 20, 2, 1, dtype=torch.float64)], -1)
    o1, l1 = oracle.fwd(q1, k1, v1, t["sinks"] + c, 0, scale)
    assert np.abs(o1[..., :8] - o0).max() < 1e-12
    assert np.abs(l1 - (l0 + c)).max() < 1e-12


def _brute(q, k, v, sinks, scale, window):
    """Separate pure-Python path: full score matrix with -inf masks, sink column appended, explicit softmax."""
    B, Lq, Hq, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    out = np.zeros((B, Lq, Hq, D))
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(Lq):
                row = []
                for j in range(Lk):
                    p = i + Lk - Lq
                    ok = (j <= p) and (window <= 0 or p - j < window)
                    row.append(scale * float(np.dot(q[b, i, h], k[b, j, g])) if ok else -math.inf)
                row.append(float(sinks[h]))
                mx = max(row)
                ex = [math.exp(x - mx) if x != -math.inf else 0.0 for x in row]
                s = sum(ex)
                for j in range(Lk):
                    out[b, i, h] += ex[j] / s * v[b, j, g]
                lse[b, h, i] = mx + math.log(s)
    return out, lse


@pytest.mark.parametrize("window", [0, 1, 3])
@pytest.mark.parametrize("Lq,Lk", [(8, 8), (5, 8), (8, 5)])
def test_brute_force_tiny(window, Lq, Lk):
    t = _inp(2, Lq, Lk, 4, 2, 4, seed=9 + Lq + Lk)
    q, k, v, s = (t[x].numpy() for x in ("q", "k", "v", "sinks"))
    bo, bl = _brute(q, k, v, s, 0.6, window)
    out, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, 0.6)
    assert np.abs(out - bo).max() < 1e-12
    assert np.abs(lse - bl).max() < 1e-12


def test_rows_without_visible_keys():
    """Lq > Lk: the first Lq - Lk rows see no key; O = 0 and LSE = sink, or
    LSE = -inf when the sink is -inf (no NaN anywhere)."""
    t = _inp(1, 10, 4, 2, 1, 4, seed=10)
    out, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 0, 0.5)
    assert np.all(out[0, :6] == 0.0)
    assert np.allclose(lse[0, :, :6], t["sinks"].numpy()[:, None], atol=0, rtol=0)
    t2 = _inp(1, 10, 4, 2, 1, 4, seed=10, sink_fill=float("-inf"), with_dout=True)
    out2, lse2 = oracle.fwd(t2["q"], t2["k"], t2["v"], t2["sinks"], 0, 0.5)
    assert np.all(out2[0, :6] == 0.0) and np.all(np.isneginf(lse2[0, :, :6]))
    assert not np.isnan(out2).any()
    dq, dk, dv, ds = oracle.bwd(t2["q"], t2["k"], t2["v"], t2["sinks"], t2["dout"], 0, 0.5)
    for a in (dq, dk, dv, ds):
        assert not np.isnan(a).any()
    assert np.all(dq[0, :6] == 0.0) and np.all(ds == 0.0)


def test_fwd_rows_matches_full():
    t = _inp(2, 40, 40, 8, 2, 16, seed=11)
    out, lse = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], 9, 0.3)
    rb = np.array([0, 1, 1, 0]); rh = np.array([0, 7, 3, 5]); ri = np.array([0, 39, 17, 8])
    o, l = oracle.fwd_rows(t["q"], t["k"], t["v"], t["sinks"], rb, rh, ri, 9, 0.3)
    for n in range(4):
        assert np.array_equal(o[n], out[rb[n], ri[n], rh[n]])
        assert l[n] == lse[rb[n], rh[n], ri[n]]


@pytest.mark.parametrize("window", [0, 6])
def test_decode_is_last_prefill_row_and_sdpa(window):
    d = decode_inputs(3, 40, 8, 2, 16, 1, 40, dtype=torch.float64, qkv_std=1.0, seed=12)
    d["sinks"] = d["sinks"].double()
    lens = d["seqlens"].tolist()
    scale = 0.25
    out, lse = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["seqlens"], d["sinks"], window, scale)
    for b, L in enumerate(lens):
        qb = d["q"][b].view(1, 1, 8, 16)
        kb = d["k_cache"][b:b + 1, :L]
        vb = d["v_cache"][b:b + 1, :L]
        ro, rl = oracle.fwd(qb, kb, vb, d["sinks"], window, scale)
        assert np.abs(out[b] - ro[0, 0]).max() < 1e-13
        assert np.abs(lse[b] - rl[0, :, 0]).max() < 1e-13
        so, sl = _sdpa_aug(qb, kb, vb, d["sinks"], scale, window)
        assert np.abs(out[b] - so[0, 0].numpy()).max() < TOL
        assert np.abs(lse[b] - sl[0, :, 0].numpy()).max() < 1e-10


@pytest.mark.parametrize("window", [0, 5])
@pytest.mark.parametrize("Lq,Lk", [(24, 24), (13, 21)])
def test_backward_matches_autograd_of_augmented_sdpa(window, Lq, Lk):
    t = _inp(2, Lq, Lk, 8, 2, 8, seed=13, with_dout=True)
    scale = 0.35
    dq, dk, dv, ds = oracle.bwd(t["q"], t["k"], t["v"], t["sinks"], t["dout"], window, scale)
    q = t["q"].clone().requires_grad_(True)
    k = t["k"].clone().requires_grad_(True)
    v = t["v"].clone().requires_grad_(True)
    s = t["sinks"].clone().requires_grad_(True)
    o, _ = _sdpa_aug(q, k, v, s, scale, window)
    (o * t["dout"]).sum().backward()
    assert np.abs(dq - q.grad.numpy()).max() < 1e-10
    assert np.abs(dk - k.grad.numpy()).max() < 1e-10
    assert np.abs(dv - v.grad.numpy()).max() < 1e-10
    assert np.abs(ds - s.grad.numpy()).max() < 1e-10


def test_backward_finite_differences():
    """Central differences of L = sum(dO * O(x)) through the oracle forward, h = 1e-6."""
    t = _inp(1, 32, 32, 4, 2, 8, seed=14, with_dout=True)
    scale, window, h = 0.3, 9, 1e-6
    dq, dk, dv, ds = oracle.bwd(t["q"], t["k"], t["v"], t["sinks"], t["dout"], window, scale)
    dO = t["dout"].numpy()

    def loss(q, k, v, s):
        o, _ = oracle.fwd(q, k, v, s, window, scale)
        return float((o * dO).sum())

    base = {x: t[x].numpy().copy() for x in ("q", "k", "v", "sinks")}
    rng = np.random.default_rng(0)

    def fd(name, idx):
        a = {x: base[x].copy() for x in base}
        a[name][idx] += h
        lp = loss(a["q"], a["k"], a["v"], a["sinks"])
        a[name][idx] -= 2 * h
        lm = loss(a["q"], a["k"], a["v"], a["sinks"])
        return (lp - lm) / (2 * h)

    for hh in range(4):
        assert abs(fd("sinks", (hh,)) - ds[hh]) <= 1e-7 * max(1.0, abs(ds[hh]))
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in base[name].shape)
            assert abs(fd(name, idx) - grad[idx]) <= 1e-7 * max(1.0, abs(grad[idx]))


def test_row_stats_reduce_to_dsink():
    t = _inp(2, 20, 20, 4, 2, 8, seed=15, with_dout=True)
    _, _, _, ds = oracle.bwd(t["q"], t["k"], t["v"], t["sinks"], t["dout"], 6, 0.4)
    Dr, Ps = oracle.row_stats(t["q"], t["k"], t["v"], t["sinks"], t["dout"], 6, 0.4)
    assert np.abs(-(Ps * Dr).sum(axis=(0, 2)) - ds).max() < 1e-12


# ----------------------------------------------------------------------------- FP8 (e4m3) K/V
def test_e4m3_values_follow_the_format():
    """The oracle's widening of E4M3 codes: closed-form values of the format
    (zero, subnormals, smallest normal, one, largest finite, NaN codes), a
    monotone order over the positive codes, and agreement with torch's
    float8_e4m3fn widening on every one of the 256 codes."""
    v = oracle.e4m3_values(np.arange(256, dtype=np.uint8))
    assert v[0x00] == 0.0 and v[0x80] == 0.0 and np.signbit(v[0x80])
    assert v[0x38] == 1.0 and v[0xB8] == -1.0
    assert v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9  # subnormals m * 2^-9
    assert v[0x08] == 2.0 ** -6 and v[0x0F] == 1.875 * 2.0 ** -6  # smallest binade of normals
    assert v[0x40] == 2.0 and v[0x3C] == 1.5
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0  # largest finite
    nan = np.isnan(v)
    assert nan[0x7F] and nan[0xFF] and nan.sum() == 2
    assert (np.diff(v[:0x7F]) > 0).all()  # positive codes in increasing order
    assert np.array_equal(v[0x80:0xFF], -v[:0x7F])  # the sign bit only flips the sign
    t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(t), nan) and np.array_equal(t[~nan], v[~nan])


def test_decode_fp8_is_decode_of_the_scaled_codes():
    """decode_fp8 = decode over code * scale per KV head: checked against the
    bf16/fp32 decode of caches widened by torch, and by two invariances of the
    scales (K's scale only rescales the logits, V's scale the output)."""
    from gqa_softmax_attention_attn_b200.inputs import quantize_e4m3_per_head

    d = decode_inputs(3, 40, 8, 2, 16, 5, 40, torch.float32, 0.5, 1.0, seed=81)
    k8, ks = quantize_e4m3_per_head(d["k_cache"])
    v8, vs = quantize_e4m3_per_head(d["v_cache"])
    kw = k8.view(torch.float8_e4m3fn).double() * ks.double()[None, None, :, None]
    vw = v8.view(torch.float8_e4m3fn).double() * vs.double()[None, None, :, None]
    for window in (0, 7):
        o, l = oracle.decode_fp8(d["q"], k8, v8, ks, vs, d["seqlens"], d["sinks"], window, 0.25)
        ro, rl = oracle.decode(d["q"], kw, vw, d["seqlens"], d["sinks"], window, 0.25)
        np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, rl, rtol=0, atol=1e-12)
        o2, l2 = oracle.decode_fp8(d["q"], k8, v8, ks * 2, vs * 4, d["seqlens"], d["sinks"], window, 0.125)
        np.testing.assert_allclose(o2, 4 * o, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(l2, l, rtol=0, atol=1e-12)


def test_fwd_fp8_is_fwd_of_the_scaled_codes():
    """fwd_fp8 = fwd over code * scale (q per query head, k and v per KV
    head): checked against the forward of inputs widened by torch's own e4m3
    cast, with per-head scales that differ (a head mapped to the wrong scale
    fails), and by the scale invariances (q's and k's scales only rescale the
    logits, v's scale the output)."""
    from gqa_softmax_attention_attn_b200.inputs import prefill_inputs, quantize_e4m3_per_head

    t = prefill_inputs(2, 24, 30, 4, 2, 16, torch.float32, 0.5, 1.0, seed=83)
    q8, qs = quantize_e4m3_per_head(t["q"] * torch.linspace(0.5, 2.0, 4)[None, None, :, None])
    k8, ks = quantize_e4m3_per_head(t["k"] * torch.tensor([1.0, 3.0])[None, None, :, None])
    v8, vs = quantize_e4m3_per_head(t["v"])
    assert len(set(qs.tolist())) == 4 and len(set(ks.tolist())) == 2
    wid = lambda c, sc: c.view(torch.float8_e4m3fn).double() * sc.double()[None, None, :, None]
    for window in (0, 5):
        o, l = oracle.fwd_fp8(q8, k8, v8, qs, ks, vs, t["sinks"], window, 0.25)
        ro, rl = oracle.fwd(wid(q8, qs), wid(k8, ks), wid(v8, vs), t["sinks"], window, 0.25)
        np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, rl, rtol=0, atol=1e-12)
        o2, l2 = oracle.fwd_fp8(q8, k8, v8, qs * 2, ks * 4, vs * 8, t["sinks"], window, 0.25 / 8)
        np.testing.assert_allclose(o2, 8 * o, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(l2, l, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- packed ragged sequences
def test_fwd_varlen_is_the_batch_when_lengths_agree_and_skips_empty_sequences():
    """fwd_varlen over B equal-length sequences packed back to back equals fwd
    on the [B, L] batch (out row for row; lse [Hq, total] = the batch's
    [B, Hq, L] laid head-major), and an empty sequence between them changes
    nothing for the others."""
    B, L, Hq, Hkv = 3, 37, 8, 2
    t = prefill_inputs(B, L, L, Hq, Hkv, 16, torch.float32, 0.5, 1.0, seed=91)
    for window in (0, 5):
        ro, rl = oracle.fwd(t["q"], t["k"], t["v"], t["sinks"], window, 0.25)
        cu = [0, L, 2 * L, 3 * L]
        o, l = oracle.fwd_varlen(t["q"].reshape(B * L, Hq, 16), t["k"].reshape(B * L, Hkv, 16),
                                 t["v"].reshape(B * L, Hkv, 16), t["sinks"], cu, cu, window, 0.25)
        assert np.array_equal(o, ro.reshape(B * L, Hq, 16))
        assert np.array_equal(l, np.concatenate(list(rl), axis=1))
        cu_e = [0, L, L, 2 * L, 3 * L]  # sequence 1 is empty
        o2, l2 = oracle.fwd_varlen(t["q"].reshape(B * L, Hq, 16), t["k"].reshape(B * L, Hkv, 16),
                                   t["v"].reshape(B * L, Hkv, 16), t["sinks"], cu_e, cu_e, window, 0.25)
        assert np.array_equal(o2, o) and np.array_equal(l2, l)


# ----------------------------------------------------------------------------- QKV prologue (YaRN rotary embedding)
YARN = dict(base=150000.0, factor=32.0, original_max_pos=4096, beta_fast=32.0, beta_slow=1.0)


def test_yarn_frequencies_closed_forms():
    """The correction dimension d(n) is where the wavelength 2 pi / f fits n
    times into L0; pairs below d(beta_fast) keep f_i exactly, pairs above
    d(beta_slow) take f_i / factor exactly, pairs between lie strictly between;
    the attention factor is 0.1 ln(factor) + 1; factor 1 is plain rotary."""
    D, base, L0 = 64, 10000.0, 4096
    f0, a0 = oracle.yarn_frequencies(D, base)
    assert a0 == 1.0 and np.array_equal(f0, base ** (-np.arange(32) * 2.0 / D))
    f, a = oracle.yarn_frequencies(D, base, 32.0, L0, 32.0, 1.0)
    lo = D * math.log(L0 / (2 * math.pi * 32.0)) / (2 * math.log(base))
    hi = D * math.log(L0 / (2 * math.pi * 1.0)) / (2 * math.log(base))
    # the wavelength at the (fractional) pair index lo fits beta_fast = 32 times into L0
    assert abs(L0 * base ** (-2 * lo / D) / (2 * math.pi) - 32.0) < 1e-9
    i = np.arange(32)
    keep, interp = i <= math.floor(lo), i >= math.ceil(hi)
    assert keep.any() and interp.any()
    assert np.array_equal(f[keep], f0[keep])
    np.testing.assert_allclose(f[interp], f0[interp] / 32.0, rtol=1e-15)
    mid = ~keep & ~interp
    assert (f[mid] < f0[mid]).all() and (f[mid] > f0[mid] / 32.0).all()
    assert abs(a - (0.1 * math.log(32.0) + 1.0)) < 1e-15
    _, a_e = oracle.yarn_frequencies(D, base, math.exp(10.0), L0)
    assert abs(a_e - 2.0) < 1e-12


@pytest.mark.parametrize("interleaved", [False, True])
def test_rotation_is_complex_multiplication(interleaved):
    """Each pair (a, b) turned by angle t is the complex number a + ib times
    attn_factor * e^{it} (written with numpy complex arithmetic here)."""
    g = np.random.default_rng(5)
    x = g.standard_normal((7, 3, 16))
    pos = g.integers(0, 131072, 7)
    f, a = oracle.yarn_frequencies(16, YARN["base"], YARN["factor"], YARN["original_max_pos"])
    r = oracle.rotate(x, pos, f, a, interleaved)
    pa, pb = (slice(0, None, 2), slice(1, None, 2)) if interleaved else (slice(0, 8), slice(8, 16))
    z = (x[..., pa] + 1j * x[..., pb]) * (a * np.exp(1j * pos[:, None, None] * f[None, None, :]))
    np.testing.assert_allclose(r[..., pa], z.real, atol=1e-12)
    np.testing.assert_allclose(r[..., pb], z.imag, atol=1e-12)


def test_rotation_depends_only_on_relative_position_and_scales_norms():
    g = np.random.default_rng(6)
    q, k = g.standard_normal((1, 1, 64)), g.standard_normal((1, 1, 64))
    f, a = oracle.yarn_frequencies(64, YARN["base"], YARN["factor"], YARN["original_max_pos"])
    dots = [float((oracle.rotate(q, [p + 1000], f, a) * oracle.rotate(k, [p], f, a)).sum()) for p in (0, 77, 50000)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)
    np.testing.assert_allclose(np.linalg.norm(oracle.rotate(q, [123456], f, a)), a * np.linalg.norm(q), rtol=1e-12)


def test_qkv_prologue_splits_adds_bias_and_rotates_q_and_k_only():
    g = np.random.default_rng(7)
    T, Hq, Hkv, D = 5, 4, 2, 16
    qkv = g.standard_normal((T, (Hq + 2 * Hkv) * D))
    bias = g.standard_normal((Hq + 2 * Hkv) * D)
    pos = g.integers(0, 5000, T)
    q, k, v = oracle.qkv_prologue(qkv, bias, pos, Hq, Hkv, D, **YARN)
    y = (qkv + bias).reshape(T, Hq + 2 * Hkv, D)
    np.testing.assert_array_equal(v, y[:, Hq + Hkv:])
    f, a = oracle.yarn_frequencies(D, **{k_: YARN[k_] for k_ in YARN if k_ != "base"}, base=YARN["base"])
    np.testing.assert_array_equal(q, oracle.rotate(y[:, :Hq], pos, f, a))
    np.testing.assert_array_equal(k, oracle.rotate(y[:, Hq:Hq + Hkv], pos, f, a))
    q0, _, _ = oracle.qkv_prologue(qkv, bias, np.zeros(T), Hq, Hkv, D, **YARN)  # position 0: scaling only
    np.testing.assert_allclose(q0, a * y[:, :Hq], rtol=1e-15)
