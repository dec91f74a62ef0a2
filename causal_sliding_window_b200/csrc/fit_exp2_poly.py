"""Coefficients of the polynomial exp2 used in the forward kernel's softmax (fwd.cuh, exp2_poly).

Method: Cody-Waite range reduction (W. J. Cody and W. Waite, "Software Manual for the Elementary
Functions", 1980): 2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]; 2^f is a
degree-3 polynomial whose coefficients minimise the maximum RELATIVE error on [-1/2, 1/2], found
with the Remez exchange algorithm (E. Ya. Remez, 1934) on the error function
e(f) = p(f) / 2^f - 1 (equioscillation at 5 points).  Run it to print the coefficients and the
error bound that the kernel's constants and the tests state.

Usage: python fit_exp2_poly.py
"""
from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg: int = DEG, iters: int = 40):
    n = deg + 2
    # Chebyshev extrema as the starting reference
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i * (-1)^i E = 2^x_i  ->  relative error alternates +-E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of err between its sign changes
        s = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(s))[0] + 1, [len(grid)]))
        ext = [lo + np.argmax(np.abs(err[lo:hi])) for lo, hi in zip(idx[:-1], idx[1:])]
        if len(ext) != n:
            break
        x = grid[ext]
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez()
    # fp32 constants as the kernel writes them
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 200001)
    e32 = float(np.max(np.abs(np.polyval(c32.astype(np.float64)[::-1], grid) / 2.0 ** grid - 1.0)))
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r}f  ({ci.view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e} (fp64 coefficients), {e32:.3e} (fp32 coefficients)")
