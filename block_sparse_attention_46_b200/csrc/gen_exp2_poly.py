"""Derives the coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on
f in [-1/2, 1/2] used by the attention kernel's FMA-pipe exponential (lf_attn.cuh,
exp2_poly).  Method: Remez exchange for the minimax RELATIVE error, in float64; the
coefficients are then rounded to float32.  Run: python gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=40):
    n = deg + 2
    k = np.arange(n)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k / (n - 1))[::-1]   # Chebyshev extrema
    grid = np.linspace(a, b, 400001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the reference points
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        segs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        while len(ext) > n:
            ext = ext[1:] if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext[:-1]
        if len(ext) == n:
            x = grid[ext]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez(deg)
    for i, v in enumerate(c):
        print(f"c{i} = {float(np.float32(v)):.9g}f")
    print(f"max relative error (exact arithmetic): {e:.3e}")
