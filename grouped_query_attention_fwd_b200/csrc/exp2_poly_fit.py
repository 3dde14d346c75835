"""Coefficients of the polynomial exp2 used on the FMA pipe by the prefill
softmax (csrc/epilogue.cuh, exp2_poly).

Method: 2^x = 2^n * 2^f with n = round-to-nearest(x) and f = x - n in
[-1/2, 1/2] (Cody and Waite style argument reduction); 2^f is replaced by the
degree-3 polynomial that minimises the maximum RELATIVE error on [-1/2, 1/2],
found with the Remez exchange algorithm (Remez 1934; see e.g. Muller,
"Elementary Functions", ch. 3).  Running this script prints the coefficients
and the error bound that the GPU test checks.
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    # Chebyshev extrema as the starting reference.
    k = np.arange(deg + 2)
    xs = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # Solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative error E).
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(xs))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # New reference: the extrema of the error between its sign changes.
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        vals = err[idx]
        # keep deg+2 alternating extrema of largest magnitude
        sel = []
        for x, v in zip(cand, vals):
            if sel and np.sign(v) == np.sign(sel[-1][1]):
                if abs(v) > abs(sel[-1][1]):
                    sel[-1] = (x, v)
            else:
                sel.append((x, v))
        while len(sel) > deg + 2:
            if abs(sel[0][1]) < abs(sel[-1][1]):
                sel.pop(0)
            else:
                sel.pop()
        xs = np.array([s[0] for s in sel])
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    for i, v in enumerate(c32):
        print("c%d = %.9ef  (%s)" % (i, v, float(v).hex()))
    print("max relative error on [-1/2, 1/2]: %.3e" % e)
