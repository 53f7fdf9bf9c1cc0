"""Fits the polynomial the kernels use for part of their exponentials.

exp2(x) is evaluated as 2^n * p(f) with n = round(x) and f = x - n in
[-1/2, 1/2] (Cody and Waite's range reduction: the power of two goes into the
exponent field, the polynomial covers one binade).  p is the degree-3
polynomial with the smallest maximum relative error to 2^f on [-1/2, 1/2],
found with the Remez exchange algorithm (equioscillation of the weighted error
at degree + 2 points), then rounded to float32.

    python exp2_poly_fit.py      prints the float32 coefficients c0..c3 and the
                                 maximum relative error of the rounded polynomial
"""

import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # start from Chebyshev extrema
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i) for the coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[: deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: the extremum of the error in each sign-alternating run
        idx = []
        sign = np.sign(err)
        start = 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or sign[k] != sign[start]:
                seg = np.arange(start, k)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = k
        if len(idx) < n:
            break
        idx = np.array(idx)
        # keep n alternating extrema with the largest magnitude
        while len(idx) > n:
            drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1
            idx = np.delete(idx, drop)
        x = grid[idx]
    return c


def max_rel_error_f32(c):
    c32 = np.asarray(c, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 1000001, dtype=np.float32)
    p = c32[3]
    for k in (2, 1, 0):
        p = (p * f + c32[k]).astype(np.float32)
    ref = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


if __name__ == "__main__":
    c = remez_relative()
    c32 = np.asarray(c, dtype=np.float32)
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v).hex()}  ({float(v):.9g})")
    print(f"max relative error (float32 Horner): {max_rel_error_f32(c32):.3e}")
