"""Coefficients of the cubic 2^f on [-1/2, 1/2] that the one-tile query x summary
kernel evaluates on the FMA pipe for a share of its exponentials.

A minimax fit of the relative error by the Remez exchange (numpy only): the
reference points start at the Chebyshev extrema, each pass solves for the
coefficients and the levelled error on them, and the next reference is the
set of alternating extrema of the error on a fine grid.  Prints the float32
coefficients and the largest relative error of their float32 Horner
evaluation, and `check()` returns both for the tests.  Used with x = n + f,
n = rint(x) added to the float's exponent field, this gives 2^x for any x the
kernel feeds it (clamped at -125 so the result stays a normal float).
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, passes: int = 30) -> np.ndarray:
    """Float64 coefficients c0..c_degree of the minimax-relative-error polynomial of 2^f."""
    n = degree + 2
    xs = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (HI - LO) / 2 + (HI + LO) / 2
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(passes):
        a = np.zeros((n, n))
        for i, x in enumerate(xs):
            a[i, :degree + 1] = [x ** k for k in range(degree + 1)]
            a[i, degree + 1] = -((-1) ** i) * np.exp2(x)
        c = np.linalg.solve(a, np.exp2(xs))[:degree + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        ext = [0]
        for i in range(1, len(grid)):
            if np.sign(err[i]) != np.sign(err[ext[-1]]):
                ext.append(i)
            elif abs(err[i]) > abs(err[ext[-1]]):
                ext[-1] = i
        if len(ext) < n:
            break
        best = max(range(len(ext) - n + 1), key=lambda s: min(abs(err[j]) for j in ext[s:s + n]))
        xs = grid[ext[best:best + n]]
    return c


def check():
    """(float32 coefficients, largest relative error of their float32 Horner evaluation on the range)."""
    c32 = remez().astype(np.float32)
    f = np.linspace(LO, HI, 2000001).astype(np.float32)
    p = np.float32(0)
    for k in range(DEGREE, -1, -1):
        p = (p * f + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    return c32, float(rel.max())


if __name__ == "__main__":
    coeffs, err = check()
    print("c0..c3 =", ", ".join(f"{float(v):.8g}f" for v in coeffs))
    print(f"largest relative error (float32 Horner): {err:.3g}")
