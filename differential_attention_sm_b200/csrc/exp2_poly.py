"""Coefficients of the cubic that approximates 2^f on [-1/2, 1/2].

The prefill kernels evaluate part of their exponentials on the FMA pipe
instead of the multi-function unit: with n = round(x) and f = x - n,
2^x = 2^n * 2^f, where 2^n is applied by adding n to the float's exponent
field and 2^f comes from this polynomial (Horner form).  The coefficients
are a minimax fit of the RELATIVE error (Remez exchange on the equioscillation
points), computed here with numpy; `python exp2_poly.py` prints them in the
form the CUDA header uses and the achieved bound.

The result only feeds probabilities that are rounded to bf16 (relative step
2^-8) before the P.V product, so a relative error near 1e-4 is far below
what the output can resolve.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _rel_err(c, x):
    return np.polynomial.polynomial.polyval(x, c) / np.exp2(x) - 1.0


def fit(degree: int = DEGREE, iters: int = 30):
    """Remez exchange for min max |p(x)/2^x - 1| over [LO, HI]."""
    n = degree + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 20001)
    c = None
    for _ in range(iters):
        # solve p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}   (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:degree + 1]
        e = _rel_err(c, grid)
        # new reference: the extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        vals = np.abs(e[idx])
        if len(cand) >= n:
            order = np.argsort(-vals)[:n]
            x = np.sort(cand[order])
    return c, float(np.abs(_rel_err(c, grid)).max())


def emulate_fp32(x: np.ndarray, c) -> np.ndarray:
    """The kernel's float32 instruction sequence, for checking its error."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    C = np.float32(12582912.0)                      # 1.5 * 2^23: round to integer
    t = (x + C).astype(np.float32)
    r = (t - C).astype(np.float32)
    f = (x - r).astype(np.float32)
    c = [np.float32(v) for v in c]
    q = (np.float32(c[3]) * f + c[2]).astype(np.float32)
    q = (q * f + c[1]).astype(np.float32)
    q = (q * f + c[0]).astype(np.float32)
    n = (t.view(np.int32) - np.array(C, np.float32).view(np.int32)).astype(np.int32)
    return (q.view(np.int32) + (n << 23)).view(np.float32)


if __name__ == "__main__":
    coef, err = fit()
    print("max relative error on [-1/2, 1/2]: %.3e" % err)
    for i, v in enumerate(coef):
        print("constexpr float kExp2C%d = %.9ef;" % (i, np.float32(v)))
    xs = np.linspace(-30.0, 8.0, 200001, dtype=np.float32)
    got = emulate_fp32(xs, coef)
    rel = np.abs(got.astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    print("float32 sequence, x in [-30, 8]: max relative error %.3e" % rel.max())
