"""Fit the polynomial the forward kernel uses for part of its exponentials.

Method: 2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody-Waite range reduction; the rounding is done by adding and subtracting
1.5 * 2^23 in fp32), and 2^f is replaced by the degree-3 polynomial that
minimises the maximum *relative* error on [-1/2, 1/2], found here with the
Remez exchange algorithm.  The kernel rounds P to bf16 (relative step 2^-8),
so a relative error near 1e-4 is far below what the result can show.

Run `python gen_exp2_poly.py` to print the coefficients and the error bound;
the printed values are the ones exp2_poly2 in sm100.cuh uses.
"""

import numpy as np


def remez_relative(degree=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    # start from Chebyshev extrema
    n = degree + 2
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :degree + 1] = xi ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        sgn = np.sign(err)
        idx = [0]
        for k in range(1, len(grid)):
            if sgn[k] != sgn[idx[-1]]:
                idx.append(k)
            elif abs(err[k]) > abs(err[idx[-1]]):
                idx[-1] = k
        if len(idx) < n:
            break
        # keep n alternating extrema with the largest |err|
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        x = grid[idx]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = [float(np.float32(v)) for v in c]
    print("coefficients c0..c3 (fp32):", ", ".join(f"{v:.9e}" for v in c32))
    g = np.linspace(-0.5, 0.5, 100001)
    p = np.polyval(np.array(c32[::-1], dtype=np.float64), g)
    print("max relative error:", float(np.max(np.abs(p / np.exp2(g) - 1))))
