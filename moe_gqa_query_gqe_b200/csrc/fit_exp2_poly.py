"""Fit the polynomial p(f) ~= 2^f on [-1/2, 1/2] used by the attention kernel's
FMA-pipe exp2 (x = j + f, 2^x = 2^j * p(f), j = round-to-nearest(x)).

Minimax in relative error by a Remez exchange on the error extrema, started
from Chebyshev nodes. Prints the coefficients (float32) and the max relative
error over a dense grid, evaluated in float32 Horner form as the kernel does.
Usage: python fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_rel(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve sum_i c_i x^i - 2^x = (-1)^k E 2^x   (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(deg + 1):
            A[:, i] = x ** i
        A[:, deg + 1] = -((-1.0) ** k) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: local extrema of err with alternating signs
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        # keep the n largest alternating extrema
        sel = []
        for i in idx:
            if sel and np.sign(err[i]) == np.sign(err[sel[-1]]):
                if abs(err[i]) > abs(err[sel[-1]]):
                    sel[-1] = i
            else:
                sel.append(i)
        while len(sel) > n:
            if abs(err[sel[0]]) < abs(err[sel[-1]]):
                sel.pop(0)
            else:
                sel.pop()
        if len(sel) < n:
            break
        x = grid[np.array(sel)]
    return c, float(np.abs(err).max())


def horner_f32(c, f):
    c32 = c.astype(np.float32)
    p = np.full_like(f, c32[-1], dtype=np.float32)
    for ci in c32[-2::-1]:
        p = (p * f + ci).astype(np.float32)
    return p


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_rel(deg)
    f = np.linspace(-0.5, 0.5, 1000001, dtype=np.float32)
    rel = np.abs(horner_f32(c, f).astype(np.float64) / 2.0 ** f.astype(np.float64) - 1).max()
    print("coefficients c0..c%d (float32):" % deg)
    for ci in c.astype(np.float32):
        print("  %.9ef" % ci)
    print("minimax rel err %.3e, float32 Horner rel err %.3e" % (e, rel))
