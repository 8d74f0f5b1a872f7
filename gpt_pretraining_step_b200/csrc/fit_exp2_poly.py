"""Coefficients of the cubic used for 2^f, |f| <= 1/2, by f2_exp2_poly in
common.cuh: a Remez exchange for the minimax *relative* error of
p(f) = c0 + c1 f + c2 f^2 + c3 f^3 against 2^f on [-1/2, 1/2].

    python fit_exp2_poly.py      # prints c0..c3 (float32) and the max relative error
"""
import numpy as np


def remez_exp2(deg=3, lo=-0.5, hi=0.5, iters=30, grid=200001):
    k = np.arange(deg + 2)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))   # Chebyshev extrema
    g = np.linspace(lo, hi, grid)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the reference points
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        c = np.linalg.solve(A, 2.0 ** x)[:deg + 1]
        err = np.polyval(c[::-1], g) / 2.0 ** g - 1
        # new reference: the extremum of each run of equal sign
        idx, start, s = [], 0, np.sign(err)
        for jj in range(1, grid + 1):
            if jj == grid or s[jj] != s[start]:
                seg = np.arange(start, jj)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = jj
        idx = np.array(idx)
        while len(idx) > deg + 2:
            idx = idx[1:] if abs(err[idx[0]]) < abs(err[idx[-1]]) else idx[:-1]
        if len(idx) == deg + 2:
            x = g[idx]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_exp2()
    print("coefficients c0..c3:", [float(np.float32(v)) for v in c])
    print("max relative error: %.3g" % e)
