"""Fit the polynomial behind the attention kernel's software base-2 exponential.

Method: Cody-Waite range reduction 2^x = 2^n * 2^f with n = rint(x) and
f = x - n in [-1/2, 1/2], then a degree-3 polynomial p(f) ~ 2^f chosen by the
Remez exchange algorithm to minimise the maximum RELATIVE error on
[-1/2, 1/2], with the constant term fixed to exactly 1 (so p(0) = 1 and the
exponent-field add never borrows below zero at the clamp x = -127).

Run:  python exp2_poly_fit.py   (prints the coefficients and the error bound;
the values are pasted into attention.cuh as kExp2C1..kExp2C3)
"""

import numpy as np


def remez_relative(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    """p(f) = 1 + c1 f + ... + c_deg f^deg minimising max |p(f)/2^f - 1| on [lo, hi]."""
    m = deg  # unknowns c1..c_deg plus the levelled error E -> deg + 1 equations
    k = np.arange(m + 1)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (m - k) / m)  # m+1 Chebyshev extrema
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # (1 + sum c_j x^j) / 2^x - 1 = (-1)^i E   ->   sum c_j x^j - (-1)^i E 2^x = 2^x - 1
        A = np.zeros((m + 1, m + 1))
        for j in range(1, deg + 1):
            A[:, j - 1] = x ** j
        A[:, m] = -((-1.0) ** np.arange(m + 1)) * np.exp2(x)
        rhs = np.exp2(x) - 1.0
        sol = np.linalg.solve(A, rhs)
        c = sol[:m]
        err = (1.0 + sum(c[j - 1] * grid ** j for j in range(1, deg + 1))) / np.exp2(grid) - 1.0
        # new reference: the extrema of the error, one per sign change interval
        idx = [0]
        for i in range(1, grid.size - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(grid.size - 1)
        idx = np.array(sorted(set(idx)))
        cand = idx[np.argsort(-np.abs(err[idx]))][: m + 1]
        x = np.sort(grid[cand])
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_relative()
    for j, cj in enumerate(c, start=1):
        print(f"c{j} = {np.float32(cj)!r}  ({cj:.17g})")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
