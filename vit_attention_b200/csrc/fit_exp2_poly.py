"""Fit the polynomial the attention kernel uses for 2^f, f in [-1/2, 1/2].

The softmax evaluates part of its exponentials on the FMA pipe instead of the
MUFU unit: 2^x = 2^j * 2^f with j = round(x), f = x - j, and 2^f from a
polynomial.  This script fits that polynomial -- minimax in relative error,
by a Remez exchange started from Chebyshev nodes -- and prints the
coefficients (low order first) and the achieved error.  Run:

    python vit_attention_b200/csrc/fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_relative(degree: int, a: float = -0.5, b: float = 0.5, iters: int = 30):
    f = lambda x: np.exp2(x)
    n = degree + 2
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n - 1 - k) / (n - 1))  # Chebyshev extrema
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # Solve p(x_i) - f(x_i) = (-1)^i E f(x_i) for the coefficients and E.
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # New reference: the extremum of the error in each sign-alternating run.
        sign = np.sign(err)
        idx = [0] + list(np.nonzero(np.diff(sign) != 0)[0] + 1) + [len(grid)]
        ext = [s + np.argmax(np.abs(err[s:e])) for s, e in zip(idx[:-1], idx[1:])]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


def fp32_error(c):
    """Max relative error of the fp32 Horner evaluation over [-1/2, 1/2]."""
    xs = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    c32 = [np.float32(v) for v in c]
    p = np.full_like(xs, c32[-1])
    for v in c32[-2::-1]:
        p = (p * xs + v).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_relative(deg)
    print("degree", deg, "minimax relative error", e, "fp32 evaluation error", fp32_error(c))
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v).item():.9e}f")
