"""Derives the polynomial the attention kernel uses for part of its exp2 work.

Method: Cody-Waite range reduction for base 2 (x = n + f with n = rint(x), so
f lies in [-1/2, 1/2] and 2^x = 2^n * 2^f exactly), then a minimax polynomial
p(f) ~ 2^f on [-1/2, 1/2] in the relative-error sense, found with the Remez
exchange algorithm (equioscillation of the weighted error at deg+2 points).

    python exp2_poly.py [degree]     # prints the coefficients c0..c_deg
"""
import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 40):
    lo, hi = -0.5, 0.5
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        f = np.exp2(x)
        # solve sum c_j x^j + (-1)^i E f(x_i) = f(x_i)  (relative-error weight 1/f)
        A = np.zeros((deg + 2, deg + 2))
        for j in range(deg + 1):
            A[:, j] = x ** j
        A[:, deg + 1] = ((-1.0) ** np.arange(deg + 2)) * f
        sol = np.linalg.solve(A, f)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: alternating extrema of the error
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = np.array(idx)
        # keep deg+2 points with alternating sign and largest magnitude
        pts = []
        for i in cand:
            if pts and np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > deg + 2:
            if abs(err[pts[0]]) < abs(err[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < deg + 2:
            break
        x = grid[pts]
    return c, np.max(np.abs(err))


def coefficients(deg: int = 3):
    c, _ = remez_exp2(deg)
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(grid)
    for cj in c32[::-1]:
        p = (p * grid + cj).astype(np.float32)
    rel = np.max(np.abs(p.astype(np.float64) - np.exp2(grid.astype(np.float64))) / np.exp2(grid.astype(np.float64)))
    return c32, float(rel)


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, rel = coefficients(deg)
    for j, cj in enumerate(c):
        print(f"c{j} = {float(cj):.9e}f  ({np.float32(cj).view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2] in fp32 Horner: {rel:.3e}")
