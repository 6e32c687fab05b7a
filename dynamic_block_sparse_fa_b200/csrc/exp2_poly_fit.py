"""Derives the polynomial used by the FMA-pipe exp2 of the prefill kernel.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (argument
reduction in the manner of Cody and Waite: the integer part goes straight
into the exponent field).  2^f is approximated on [-1/2, 1/2] by a cubic
chosen to minimise the maximum relative error (Remez exchange started from
Chebyshev nodes).  Prints the coefficients (constant term first) and the
achieved maximum relative error.

    python dynamic_block_sparse_fa_b200/csrc/exp2_poly_fit.py
"""
import numpy as np


def remez_relative(deg=3, a=-0.5, b=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [grid.size]])
        xs = []
        for s0, s1 in zip(bounds[:-1], bounds[1:]):
            seg = np.arange(s0, s1)
            xs.append(grid[seg[np.argmax(np.abs(err[seg]))]])
        if len(xs) == n:
            x = np.array(xs)
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez_relative()
    print("coefficients (c0..c3):", ", ".join(f"{v:.9e}" for v in c))
    print("max relative error on [-1/2, 1/2]:", f"{e:.3e}")
    # in float32 as the kernel evaluates it (Horner, FMA)
    c32 = c.astype(np.float32)
    xs = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.full_like(xs, c32[3])
    for ci in c32[2::-1]:
        p = (p * xs + ci).astype(np.float32)
    print("float32 evaluation max relative error:",
          f"{np.abs(p / np.exp2(xs.astype(np.float64)) - 1).max():.3e}")
