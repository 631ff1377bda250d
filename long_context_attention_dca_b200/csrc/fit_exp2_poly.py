"""Refit the exp2 polynomial of exp2_poly.cuh (not run at build time).

Remez exchange for the degree-d polynomial p minimising the maximum relative
error |p(f) - 2^f| / 2^f on f in [-1/2, 1/2]; prints the coefficients c0..cd
rounded to fp32 and the maximum relative error of their fp32 Horner
evaluation.  exp2_poly.cuh uses d = 3.
"""

import sys

import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        segs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segs]
        while len(ext) > n:
            ext = ext[1:] if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext[:-1]
        if len(ext) == n:
            x = grid[ext]
    return c


def fp32_horner_error(c):
    c32 = np.asarray(c, np.float32)
    t = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.full_like(t, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * t + c32[k]).astype(np.float32)
    ref = np.exp2(t.astype(np.float64))
    return float(np.max(np.abs(p - ref) / ref))


if __name__ == "__main__":
    d = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez(d)
    print([float(np.float32(v)) for v in c], "max rel err (fp32):", fp32_horner_error(c))
