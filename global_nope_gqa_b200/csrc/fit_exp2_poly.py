"""Fit the cubic that the prefill kernel uses for part of its exp2 evaluations.

2^y = 2^k * 2^f with k = round(y) and f = y - k in [-1/2, 1/2].  The cubic
c0 + c1 f + c2 f^2 + c3 f^3 approximates 2^f on that interval with the least
maximum relative error (Remez exchange on the relative error, from Chebyshev
nodes).  Run this file to print the coefficients written into prefill_tc.cuh
and the error bound the CPU test checks.
"""
import numpy as np


def remez_relative(deg=3, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve sum c_i x^i - f(x) = (-1)^j E f(x)  (relative equioscillation)
        A = np.zeros((n, n))
        for j in range(n):
            A[j, :deg + 1] = x[j] ** np.arange(deg + 1)
            A[j, deg + 1] = -((-1) ** j) * f(x[j])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        grid = np.linspace(a, b, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of err between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        # keep n alternating extrema of largest magnitude
        best = []
        for i in idx:
            if best and np.sign(err[i]) == np.sign(err[best[-1]]):
                if abs(err[i]) > abs(err[best[-1]]):
                    best[-1] = i
            else:
                best.append(i)
        while len(best) > n:
            if abs(err[best[0]]) < abs(err[best[-1]]):
                best.pop(0)
            else:
                best.pop()
        if len(best) == n:
            x = grid[best]
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = ((c32[3] * grid + c32[2]) * grid + c32[1]) * grid + c32[0]
    e32 = np.max(np.abs(p.astype(np.float64) / np.exp2(grid.astype(np.float64)) - 1))
    print("coefficients (c0..c3):", ", ".join(f"{float(v):.9e}f" for v in c32))
    print(f"max relative error: {e:.3e} (double coefficients), {e32:.3e} (float32 Horner)")
