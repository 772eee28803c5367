"""Fits the polynomial the attention kernel uses for part of its exp2 calls.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody and Waite's argument reduction); 2^f is approximated by a degree-3
polynomial p(f) that minimises the maximum relative error |p(f)/2^f - 1| on
[-1/2, 1/2], found with the Remez exchange algorithm (equioscillation on
deg + 2 points). The kernel rounds p(f) to bf16/fp16 afterwards (relative
step 2^-9 / 2^-11), so a relative error near 1e-4 is well inside that.

Run:  python fit_exp2_poly.py   -> prints the coefficients c0..c3 and the error.
"""

import numpy as np


def remez_relative(func, deg, lo, hi, iters=30):
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i * E * f(x_i)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * func(x[i])
        sol = np.linalg.solve(A, func(x))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / func(grid) - 1.0
        # new reference: extrema of err between sign changes
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        # keep the n largest alternating extrema
        cand = sorted(idx, key=lambda j: -abs(err[j]))
        chosen = []
        for j in sorted(cand[: 4 * n]):
            if chosen and np.sign(err[j]) == np.sign(err[chosen[-1]]):
                if abs(err[j]) > abs(err[chosen[-1]]):
                    chosen[-1] = j
            else:
                chosen.append(j)
        if len(chosen) < n:
            break
        while len(chosen) > n:
            if abs(err[chosen[0]]) < abs(err[chosen[-1]]):
                chosen.pop(0)
            else:
                chosen.pop()
        x = grid[chosen]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    coeffs, max_rel = remez_relative(lambda t: np.exp2(t), 3, -0.5, 0.5)
    for i, c in enumerate(coeffs):
        print(f"c{i} = {np.float32(c)!r}  ({c:.17g})")
    print(f"max relative error = {max_rel:.3e}")
