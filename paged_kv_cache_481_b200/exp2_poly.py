"""Coefficients of the polynomial 2^x that the prefill softmax evaluates on
the FMA pipes for part of its scores.

    python -m paged_kv_cache_481_b200.exp2_poly

Method: Cody-Waite range reduction x = j + f with j = floor(x) (exact in
fp32), 2^x = 2^j * 2^f, and a degree-3 polynomial p(f) ~ 2^f on [0, 1)
minimising the maximum RELATIVE error (Remez exchange on the equioscillation
points).  2^j enters by adding j to the exponent field of p(f).  The result
only feeds an fp16 rounding of the attention weight (relative step 2^-11),
so a relative error near 1e-4 is invisible at the output.

This module only derives and checks the numbers; the kernel carries them as
constants (kExp2C0..kExp2C3 in csrc/prefill_kernel.cuh) and
tests/test_exp2_poly.py checks that the two agree and that the fp32 Horner
evaluation stays within the error bound.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def _solve(points):
    """Coefficients c0..cD and level E with p(x_i) / 2^x_i - 1 = (-1)^i E."""
    n = DEGREE + 2
    a = np.zeros((n, n))
    rhs = np.zeros(n)
    for i, x in enumerate(points):
        t = 2.0 ** x
        a[i, :DEGREE + 1] = [x ** k / t for k in range(DEGREE + 1)]
        a[i, DEGREE + 1] = -((-1) ** i)
        rhs[i] = 1.0
    sol = np.linalg.solve(a, rhs)
    return sol[:DEGREE + 1], sol[DEGREE + 1]


def fit(iterations: int = 30):
    """Remez exchange for the relative error of p(f) against 2^f on [0, 1]."""
    n = DEGREE + 2
    pts = 0.5 - 0.5 * np.cos(np.pi * np.arange(n) / (n - 1))   # Chebyshev start
    grid = np.linspace(0.0, 1.0, 200001)
    for _ in range(iterations):
        c, _ = _solve(pts)
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign run of the error
        sign = np.sign(err)
        cuts = np.flatnonzero(np.diff(sign)) + 1
        runs = np.split(np.arange(grid.size), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < n:
            break
        # keep the n largest alternating extrema
        while len(ext) > n:
            mags = np.abs(err[ext])
            drop = 0 if mags[0] < mags[-1] else len(ext) - 1
            ext.pop(drop)
        pts = grid[ext]
    c, _ = _solve(pts)
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.max(np.abs(err)))


def horner_fp32(c, f):
    """p(f) evaluated as the kernel does: fp32 Horner with fused multiply-adds
    (each step rounded once, emulated in float64 then rounded to fp32)."""
    c32 = np.asarray(c, dtype=np.float32)
    f32 = np.asarray(f, dtype=np.float32).astype(np.float64)
    acc = np.float64(c32[DEGREE])
    for k in range(DEGREE - 1, -1, -1):
        acc = (acc * f32 + np.float64(c32[k])).astype(np.float32).astype(np.float64)
    return acc


if __name__ == "__main__":
    coeffs, max_rel = fit()
    for k, v in enumerate(coeffs):
        print(f"c{k} = {np.float32(v)!r}  ({v:.17g})")
    print(f"max relative error on [0, 1]: {max_rel:.3e}")
