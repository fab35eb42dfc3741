"""Fits the polynomial used for 2^f on f in [-1/2, 1/2] by the attention
kernels' FMA-pipe exponential (Cody-Waite style reduction x = n + f, n the
nearest integer, 2^x = 2^n * p(f)).  Minimax in relative error by Remez
exchange on p(f) / 2^f - 1, run in float64 with numpy.  Prints the
coefficients c0..cD (p(f) = c0 + c1 f + ... + cD f^D) and the max relative
error of the fit.  Usage: python fit_exp2_poly.py [degree]."""
import sys

import numpy as np


def remez(deg, iters=30):
    lo, hi = -0.5, 0.5
    m = deg + 2
    k = np.arange(m)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (m - 1 - k) / (m - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve c_j x_i^j - E (-1)^i 2^{x_i} = 2^{x_i}  (relative error alternation)
        A = np.zeros((m, m))
        for i in range(m):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if s[i] != s[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        idx = np.array(idx)
        if len(idx) >= m:
            best = None
            for start in range(len(idx) - m + 1):
                cand = idx[start:start + m]
                v = np.min(np.abs(err[cand]))
                if best is None or v > best[0]:
                    best = (v, cand)
            x = grid[best[1]]
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez(deg)
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v)!r}  ({v:.17g})")
    print(f"max relative error {e:.3e}")
