"""The oracle's pins must catch plausible mistakes (CPU only).

Each case plants one mistake in a private copy of the C oracle, compiles it,
and checks that at least one pin in test_oracle_pins.py fails against it.
Nothing here touches a GPU.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_sink_oracle.c")

MUTANTS = {
    "sink-mass-dropped": ("double Z = exp(sink - M);", "double Z = 0.0 * exp(sink - M);"),
    "sink-scaled": ("double Z = exp(sink - M);", "double Z = exp(0.5 * sink - M);"),
    "window-off-by-one": ("if (window > 0 && j <= p - window) return 0;", "if (window > 0 && j < p - window) return 0;"),
    "gqa-mapping": ("const int g = h / G;\n        const double *qi = q + (((long)b * Lq + i) * Hq + h) * D;\n        const double *kb",
                    "const int g = h % Hkv;\n        const double *qi = q + (((long)b * Lq + i) * Hq + h) * D;\n        const double *kb"),
    "value-from-key": ("const double *vj = v0 + j * row_stride;", "const double *vj = k0 + j * row_stride;"),
    "causal-top-left": ("fwd_row(qi, kb, vb, (long)Hkv * D, Lk, (long)i + (Lk - Lq), window, scale, sinks[h],\n                D, oi,",
                        "fwd_row(qi, kb, vb, (long)Hkv * D, Lk, (long)i, window, scale, sinks[h],\n                D, oi,"),
    "ds-sign": ("const double dS = P * (dot(doi, vj, D) - Di);", "const double dS = P * (dot(doi, vj, D) + Di);"),
    "dsink-sign": ("s -= Ps[r] * Dr[r];", "s += Ps[r] * Dr[r];"),
    "dk-unscaled": ("dkj[d] += scale * dS * qi[d];", "dkj[d] += dS * qi[d];"),
    "lse-without-log": ("*lse = M + log(Z);", "*lse = M + Z;"),
}

PIN_BATTERY = [
    lambda: pins.test_matches_augmented_sdpa(5, 40, 40, 8, 2),
    lambda: pins.test_matches_augmented_sdpa(0, 17, 30, 4, 4),
    lambda: pins.test_sink_neg_inf_is_plain_causal_gqa_sdpa(20, 47),
    lambda: pins.test_window_one_closed_form(),
    lambda: pins.test_backward_matches_autograd_of_augmented_sdpa(5, 24, 24),
    lambda: pins.test_row_mass_plus_sink_mass_is_one(7),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    c = tmp_path / "mutant.c"
    c.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-o", str(so), str(c), "-lm"])
    caught = []
    with oracle.use_library(str(so)):
        for pin in PIN_BATTERY:
            try:
                pin()
            except AssertionError:
                caught.append(pin)
    assert caught, f"no pin caught the planted mistake '{name}'"
