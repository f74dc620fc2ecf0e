"""Fits the polynomial used by the kernels' software exp2 (fast_exp2 in sm100_ptx.cuh).

Method: range reduction x = n + f with n = round(x), f in [-1/2, 1/2]
(Cody-Waite style, exact in fp32 for |x| < 2^22), then 2^f ~ p(f) with p the
minimax polynomial for the RELATIVE error on [-1/2, 1/2], found by a Remez
exchange; 2^x = p(f) * 2^n is assembled by adding n to the exponent field.

Run: python exp2_poly.py [degree]   (prints the coefficients as fp32 literals
and the achieved max relative error, measured in fp32 arithmetic.)
"""
import sys

import numpy as np


def remez_rel(deg, lo=-0.5, hi=0.5, iters=40):
    n = deg + 2
    # Chebyshev points as the initial reference
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (equi-oscillating relative error)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = np.where(np.diff(s) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) < n:
            break
        # keep the n largest alternating extrema
        ext = np.array(ext)
        while len(ext) > n:
            drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else len(ext) - 1
            ext = np.delete(ext, drop)
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


def fp32_eval_error(c):
    """Max relative error of the full fp32 evaluation path over a dense grid of x in [-30, 8]."""
    c32 = [np.float32(v) for v in c]
    xs = np.linspace(-30.0, 8.0, 2000001).astype(np.float32)
    magic = np.float32(12582912.0)
    t = (xs + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    fr = (xs - r).astype(np.float32)
    p = np.float32(c32[-1])
    for cc in reversed(c32[:-1]):
        p = (p * fr + cc).astype(np.float32)
    n = r.astype(np.int64)
    val = p.astype(np.float64) * np.exp2(n.astype(np.float64))
    ref = np.exp2(xs.astype(np.float64))
    return float(np.max(np.abs(val / ref - 1)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_rel(deg)
    print(f"degree {deg}: minimax relative error {e:.3e}; fp32 path max relative error {fp32_eval_error(c):.3e}")
    for i, v in enumerate(c):
        print(f"  c{i} = {float(np.float32(v)):.9g}f")
