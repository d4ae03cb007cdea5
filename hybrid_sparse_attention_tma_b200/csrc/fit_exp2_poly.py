"""Fit the degree-3 polynomial used by the FMA-pipe exp2 in the softmax.

Method: Cody-Waite style range reduction (x = j + f, j = round(x),
f in [-1/2, 1/2]) followed by a minimax polynomial p(f) ~ 2^f that minimises
the maximum RELATIVE error on [-1/2, 1/2]; 2^x = p(f) * 2^j, the 2^j applied
by adding j to the float's exponent field. The minimax fit is a plain Remez
exchange on the weighted error (p(f) - 2^f) / 2^f.

Run: python fit_exp2_poly.py  -> prints the coefficients c0..c3 and the
maximum relative error; the values are pasted into hs_common.cuh.
"""
import numpy as np


def remez(deg=3, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    ref = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    f = lambda x: np.exp2(x)  # noqa: E731
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative weighting)
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of the error
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        vals = err[idx]
        # keep n points with alternating signs and largest magnitude
        pts = []
        for x, v in zip(cand, vals):
            if pts and np.sign(v) == np.sign(pts[-1][1]):
                if abs(v) > abs(pts[-1][1]):
                    pts[-1] = (x, v)
            else:
                pts.append((x, v))
        while len(pts) > n:
            if abs(pts[0][1]) < abs(pts[-1][1]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) == n:
            ref = np.array([x for x, _ in pts])
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez()
    print("coefficients c0..c3:", ", ".join(f"{x:.9e}" for x in c))
    print("max relative error:", e)
    c32 = c.astype(np.float32).astype(np.float64)
    g = np.linspace(-0.5, 0.5, 1000001)
    print("max relative error with fp32 coefficients:",
          np.abs((np.polyval(c32[::-1], g) - np.exp2(g)) / np.exp2(g)).max())
