"""Fit the polynomial used by the FMA-pipe exp2 in sm100.cuh.

Method: Cody–Waite style range reduction, x = n + f with n = round(x) and
f in [-1/2, 1/2], so 2^x = 2^n * 2^f; 2^n is applied by adding n to the float
exponent field, 2^f is a polynomial P(f) = sum_k c_k f^k whose coefficients
minimise the maximum RELATIVE error |P(f) / 2^f - 1| on [-1/2, 1/2] (a Remez
exchange on the Haar system {f^k}, weight 1/2^f). Run:

    python gen_exp2_poly.py [degree]

and paste the printed coefficients (float32) into sm100.cuh.
"""
import sys

import numpy as np


def remez(degree: int, lo=-0.5, hi=0.5, iters=60):
    n = degree + 1
    # start from Chebyshev extrema
    k = np.arange(n + 1)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k / n)[::-1]
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve sum c_j x_i^j - f(x_i) = (-1)^i E f(x_i)  (relative error alternation)
        A = np.zeros((n + 1, n + 1))
        for i, xi in enumerate(x):
            A[i, :n] = xi ** np.arange(n)
            A[i, n] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c, E = sol[:n], sol[n]
        grid = np.linspace(lo, hi, 20001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of err between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        cerr = err[idx]
        # keep n+1 alternating points with the largest |err|
        pts = []
        for xi, ei in zip(cand, cerr):
            if pts and np.sign(ei) == np.sign(pts[-1][1]):
                if abs(ei) > abs(pts[-1][1]):
                    pts[-1] = (xi, ei)
            else:
                pts.append((xi, ei))
        while len(pts) > n + 1:
            if abs(pts[0][1]) < abs(pts[-1][1]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < n + 1:
            break
        x = np.array([p[0] for p in pts])
    grid = np.linspace(lo, hi, 200001)
    c32 = c.astype(np.float32).astype(np.float64)
    err = np.abs((np.polyval(c32[::-1], grid) - f(grid)) / f(grid)).max()
    return c.astype(np.float32), err


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, err = remez(deg)
    print(f"degree {deg}: max relative error {err:.3e} on [-0.5, 0.5]")
    for i, v in enumerate(c):
        print(f"  c{i} = {float(v):.9e}f")
