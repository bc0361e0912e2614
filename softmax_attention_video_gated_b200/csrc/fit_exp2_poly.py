"""Fits the cubic used by the softmax anchor to evaluate part of its
exponentials on the FMA pipe instead of the MUFU unit.

Method: Cody-Waite range reduction 2^x = 2^n * 2^f with n = rint(x) and
f = x - n in [-1/2, 1/2], then a minimax polynomial p(f) ~ 2^f (relative
error, equioscillation by the Remez exchange algorithm) of degree 3. The
constant term is pinned to 1 so 2^0 is exact. Run this file to reproduce
the coefficients printed into anchor_tc.cu and the error bound.
"""
import numpy as np


def remez(deg=3, iters=30):
    # unknowns: c1..c_deg and the levelled error E; c0 = 1
    lo, hi = -0.5, 0.5
    k = deg + 1  # number of alternation points
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(k) / (k - 1))[::-1]
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  with p(x) = 1 + sum c_j x^j
        A = np.zeros((k, deg + 1))
        b = np.zeros(k)
        for i, xi in enumerate(x):
            t = 2.0 ** xi
            A[i, :deg] = [xi ** j for j in range(1, deg + 1)]
            A[i, deg] = -((-1) ** i) * t
            b[i] = t - 1.0
        sol = np.linalg.solve(A, b)
        c = np.concatenate([[1.0], sol[:deg]])
        grid = np.linspace(lo, hi, 200001)
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new alternation points: extrema of err between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = sorted(idx, key=lambda i: -abs(err[i]))[:k]
        x = np.sort(grid[cand])
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez()
    print("coefficients c0..c3:", ", ".join(repr(float(np.float32(v))) for v in c))
    print("max relative error on [-1/2, 1/2]:", e)
