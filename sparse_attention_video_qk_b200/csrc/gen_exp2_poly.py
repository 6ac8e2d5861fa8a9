"""Coefficients of the polynomial exp2 used by the attention softmax.

2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2].  2^f is
approximated by a degree-`deg` polynomial whose coefficients minimise the
maximum *relative* error on [-1/2, 1/2] (Remez exchange algorithm on the
weighted error (p(f) - 2^f) / 2^f), with p(0) free.  Run:

    python gen_exp2_poly.py [deg]

and copy the printed constants (rounded to fp32) into attention.cuh.
"""
import sys

import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=60):
    f = lambda x: np.exp2(x)
    n = deg + 2
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))   # Chebyshev extrema
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error with alternating sign
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(sorted(set(idx)))
        # keep the n largest alternating extrema
        cand = idx[np.argsort(-np.abs(err[idx]))]
        chosen = sorted(cand[:n])
        if len(chosen) == n:
            x = grid[chosen]
    return c, np.abs(err).max()


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez(deg)
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 100001)
    e32 = np.abs((np.polyval(c32[::-1].astype(np.float64), g) - np.exp2(g)) / np.exp2(g)).max()
    print(f"degree {deg}: max relative error {e:.3e} (fp32 coefficients: {e32:.3e})")
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v)!r}f")
