"""Fit the degree-3 polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the
attention kernel's FMA-pipe exp2 (Cody-Waite reduction x = j + f, j the
nearest integer, then 2^x = 2^j * p(f)).

The fit minimises the maximum relative error with a Remez exchange on the
equioscillation of p(f) * 2^-f - 1, starting from Chebyshev nodes.  Run it
to print the coefficients that attn_sm100.cu embeds and the error bound.
"""
import numpy as np


def fit(deg=3, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n) / (n - 1))[::-1]
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i * E * 2^x_i  (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error, one per sign run
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = sorted(idx, key=lambda i: -abs(err[i]))
        keep = sorted(idx[:n])
        x = grid[keep]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = fit()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = p * grid + np.float32(c32[k])
    e32 = float(np.max(np.abs(p.astype(np.float64) / 2.0 ** grid.astype(np.float64) - 1.0)))
    print("coefficients c0..c3 (fp32):", ", ".join("%.9ef" % v for v in c32))
    print("max relative error: fit %.3e, evaluated in fp32 %.3e" % (e, e32))
