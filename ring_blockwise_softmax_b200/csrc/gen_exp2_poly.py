"""Derive the coefficients of exp2_poly3 (ra_fmha_sm100.cuh).

2^f on [-1/2, 1/2] by a degree-3 polynomial that is minimax in *relative* error, found with the
Remez exchange algorithm: solve p(x_i) + (-1)^i E 2^{x_i} = 2^{x_i} on n = deg + 2 reference
points, move the references to the alternating extrema of the weighted error, repeat.  Prints
the coefficients rounded to fp32 (lowest order first) and the resulting maximum relative error.

    python ring_blockwise_softmax_b200/csrc/gen_exp2_poly.py
"""

import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[: deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        idx = [0]
        for k in range(1, grid.size):
            if np.sign(err[k]) != np.sign(err[idx[-1]]):
                idx.append(k)
            elif abs(err[k]) > abs(err[idx[-1]]):
                idx[-1] = k
        idx = np.array(idx)
        if idx.size >= n:
            best = max(range(idx.size - n + 1), key=lambda s0: np.min(np.abs(err[idx[s0:s0 + n]])))
            x = grid[idx[best:best + n]]
    return c


if __name__ == "__main__":
    c32 = remez(3).astype(np.float32)
    g = np.linspace(-0.5, 0.5, 1000001)
    e = np.max(np.abs((np.polyval(c32[::-1].astype(np.float64), g) - np.exp2(g)) / np.exp2(g)))
    print("coefficients (c0..c3):", [float(v) for v in c32])
    print("max relative error:", e)
