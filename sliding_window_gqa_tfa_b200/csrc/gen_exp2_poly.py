"""Fit the polynomial the kernel uses for 2^f on f in [-1/2, 1/2].

Method: Cody-Waite argument reduction (2^x = 2^n * 2^f with n = round(x),
f = x - n) leaves 2^f on a half-unit interval; the polynomial is the
relative-error minimax of the given degree there, found with the Remez exchange
algorithm (equioscillation of the weighted error (p(f) - 2^f) / 2^f at
degree + 2 points), in float64.  Printed as float32 literals for
tfa_ptx.cuh.

    python sliding_window_gqa_tfa_b200/csrc/gen_exp2_poly.py [degree]
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(degree: int, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    n = degree + 2
    # initial reference: Chebyshev extrema mapped to [lo, hi]
    k = np.arange(n)
    xs = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  for the coefficients and E
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** xs)
        coef = sol[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extrema of the error between sign changes
        sign = np.sign(err)
        idx = np.concatenate([[0], np.nonzero(np.diff(sign))[0] + 1, [grid.size]])
        ext = [seg_lo + np.argmax(np.abs(err[seg_lo:seg_hi]))
               for seg_lo, seg_hi in zip(idx[:-1], idx[1:]) if seg_hi > seg_lo]
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest magnitude
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        xs = grid[ext]
    err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
    return coef, float(np.max(np.abs(err)))


def float32_error(coef32, lo=-0.5, hi=0.5):
    """Max relative error of the Horner evaluation in float32 (fma-free bound)."""
    f = np.linspace(lo, hi, 100001).astype(np.float32)
    p = np.float32(coef32[-1])
    for c in coef32[-2::-1]:
        p = (p * f + np.float32(c)).astype(np.float32)
    return float(np.max(np.abs((p.astype(np.float64) - 2.0 ** f.astype(np.float64)) /
                               2.0 ** f.astype(np.float64))))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_exp2(deg)
    c32 = [np.float32(x) for x in c]
    print(f"// degree {deg}: minimax relative error {e:.3e} (float64), "
          f"{float32_error(c32):.3e} evaluated in float32")
    for i, x in enumerate(c32):
        print(f"constexpr float kExp2C{i} = {float(x)!r}f;")
