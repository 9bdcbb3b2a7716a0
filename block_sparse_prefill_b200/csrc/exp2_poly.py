"""Coefficients of the polynomial exp2 used by the attention kernel.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is
approximated by the degree-3 polynomial p(f) = c0 + c1 f + c2 f^2 + c3 f^3
that minimises the maximum RELATIVE error on [-1/2, 1/2], found with the
Remez exchange algorithm (alternation of the weighted error at n + 2 points).
Run this file to regenerate the constants in attention.cu.
"""
import numpy as np


def remez_exp2(deg=3, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    # Chebyshev points as the initial reference
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    f = lambda t: np.exp2(t)
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)   (relative error weight 1/f)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c, E = sol[:deg + 1], sol[deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: the extrema of the error on each sign interval
        idx = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_exp2()
    c32 = np.float32(c)
    grid = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = ((c32[3] * grid + c32[2]) * grid + c32[1]) * grid + c32[0]
    e32 = float(np.abs(p.astype(np.float64) / np.exp2(grid.astype(np.float64)) - 1).max())
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v):.9e}f  (0x{np.float32(v).view(np.uint32):08x})")
    print(f"max relative error: {e:.3e} (fp64 coefficients), {e32:.3e} (fp32 Horner)")
