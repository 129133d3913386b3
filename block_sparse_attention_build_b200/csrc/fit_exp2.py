"""Fit the polynomial the forward kernel uses for part of its exponentials.

The kernel splits 2^x as 2^j * 2^f with j = round(x) and f in [-1/2, 1/2]
(Cody-Waite range reduction with a single exact step, since the split of a
binary exponent is exact), puts j into the exponent field, and approximates
2^f by a polynomial.  This script finds the polynomial of the given degree
that minimises the maximum RELATIVE error on [-1/2, 1/2] (Remez exchange on
the weighted error (p(f) - 2^f) / 2^f), then reports that error and the error
of the same polynomial evaluated in float32 with fused multiply-adds.

Run:  python fit_exp2.py [degree]   (prints coefficients c0..cd, lowest first)
"""
from __future__ import annotations

import sys

import numpy as np


def remez(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 40):
    """Minimax relative-error fit of 2^f on [a, b] by the Remez exchange."""
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(a, b, 20001)
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E 2^{x_i} = 2^{x_i}
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c, E = sol[: deg + 1], sol[deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of the error
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        ext = grid[idx]
        vals = err[idx]
        # keep n points with alternating signs and largest magnitude
        pts = []
        for xi, vi in zip(ext, vals):
            if pts and np.sign(vi) == np.sign(pts[-1][1]):
                if abs(vi) > abs(pts[-1][1]):
                    pts[-1] = (xi, vi)
            else:
                pts.append((xi, vi))
        while len(pts) > n:
            pts.pop(0 if abs(pts[0][1]) < abs(pts[-1][1]) else -1)
        if len(pts) < n:
            break
        x = np.array([p_[0] for p_ in pts])
    return c, np.abs(err).max()


def float32_error(c, a=-0.5, b=0.5):
    """Max relative error of Horner evaluation in float32 with fused multiply-add
    (each step rounded once), against 2^f in float64."""
    cs = [np.float32(v) for v in c]
    t = np.linspace(a, b, 200001).astype(np.float32)
    acc = np.full_like(t, cs[-1])
    for cc in reversed(cs[:-1]):
        acc = (acc.astype(np.float64) * t.astype(np.float64) + np.float64(cc)).astype(np.float32)
    ref = np.exp2(t.astype(np.float64))
    return float(np.abs((acc.astype(np.float64) - ref) / ref).max())


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c, e = remez(deg)
    print(f"degree {deg}: minimax relative error {e:.3e}, float32 evaluation {float32_error(c):.3e}")
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v).item()!r}f  // {v!r}")
