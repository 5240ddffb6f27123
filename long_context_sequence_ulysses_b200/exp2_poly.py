"""Coefficients of the FMA-pipe exp2 used by the attention softmax.

The kernels evaluate part of their exponentials without the special-function
unit, by the classic range reduction (Cody and Waite, "Software Manual for the
Elementary Functions", 1980): 2^x = 2^j * 2^f with j = round(x) and
f = x - j in [-1/2, 1/2], where 2^f is a polynomial and 2^j is added into the
exponent field. The polynomial is the degree-3 minimax approximation of 2^f on
[-1/2, 1/2] in relative error, found here with the Remez exchange algorithm,
then rounded to fp32.

    python -m long_context_sequence_ulysses_b200.exp2_poly   # prints the coefficients

The fp32 values are written into csrc/ptx.cuh (ex2_poly); a test checks that
they match this script and bounds the error of the whole device algorithm.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_exp2(degree: int = DEGREE, iters: int = 30):
    """Minimax polynomial for 2^f on [LO, HI] in relative error."""
    n = degree + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))   # Chebyshev extrema
    grid = np.linspace(LO, HI, 200001)
    target = np.exp2(grid)
    coeffs = None
    for _ in range(iters):
        # Solve p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i} for the coefficients and E.
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        coeffs = sol[:degree + 1]
        err = (np.polyval(coeffs[::-1], grid) - target) / target
        # new reference: the extrema of the error, one per sign change interval
        d = np.diff(err)
        turn = np.nonzero(d[:-1] * d[1:] <= 0)[0] + 1
        idx = np.unique(np.concatenate([[0], turn, [len(grid) - 1]]))
        cand = idx[np.argsort(-np.abs(err[idx]))]
        pts = []
        for c in cand:
            if all(abs(grid[c] - grid[p]) > 1e-3 for p in pts):
                pts.append(c)
            if len(pts) == n:
                break
        x = np.sort(grid[np.array(pts)])
    return coeffs


def fp32_coefficients():
    return np.asarray(remez_exp2(), dtype=np.float32)


def emulate(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The device algorithm, step by step in fp32 (round-to-nearest)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)                      # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    fi = (t - magic).astype(np.float32)
    f = (x - fi).astype(np.float32)
    p = np.float32(c[3])
    p = (p * f + np.float32(c[2])).astype(np.float32)   # fmaf rounding differs by < 1 ulp from this
    p = (p * f + np.float32(c[1])).astype(np.float32)
    p = (p * f + np.float32(c[0])).astype(np.float32)
    j = t.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (j << 23)).view(np.float32)


if __name__ == "__main__":
    c = fp32_coefficients()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}  ({v.view(np.uint32):#010x})")
    xs = np.linspace(-30, 8, 1000001, dtype=np.float32)
    rel = np.abs(emulate(xs, c).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1)
    print("max relative error on [-30, 8]:", rel.max())
