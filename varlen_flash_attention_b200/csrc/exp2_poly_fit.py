"""Fit the polynomial used for exp2 on the FMA pipe in the attention softmax.

Method (Cody-Waite range reduction, then a minimax fit):
  x = n + f with n = round-to-nearest(x), f in [-1/2, 1/2]
  2^x = 2^n * p(f),  p(f) ~= 2^f
p is the degree-3 polynomial that minimises the maximum relative error on
[-1/2, 1/2], found by a Remez exchange on the relative error.  Its coefficients are rounded to fp32 and the resulting error is
reported.  The kernel rounds p to bf16 afterwards (relative step 2^-8), so an
error well below 2^-9 is invisible in P.

Run: python exp2_poly_fit.py  (prints the fp32 coefficients and the error)
"""
import numpy as np


def fit(deg=3, iters=30):
    # p(f) = c0 + c1 f + ... + c_deg f^deg ; minimise max |p(f)/2^f - 1|
    a, b = -0.5, 0.5
    m = deg + 1  # unknowns c0..c_deg plus the level E -> deg + 2 equations
    # initial reference points: Chebyshev extrema
    k = np.arange(m + 1)
    xs = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k / m)[::-1]
    for _ in range(iters):
        A = np.zeros((m + 1, m + 1))
        rhs = np.zeros(m + 1)
        for i, x in enumerate(xs):
            t = 2.0 ** x
            for j in range(m):
                A[i, j] = x ** j / t
            A[i, m] = (-1.0) ** i
            rhs[i] = 1.0
        sol = np.linalg.solve(A, rhs)
        c = sol[:m]
        grid = np.linspace(a, b, 200001)
        err = sum(c[j] * grid ** j for j in range(m)) / 2.0 ** grid - 1.0
        # new reference: extrema of err in m+1 alternating segments
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = sorted(set(idx), key=lambda i: grid[i])
        pts = sorted(idx, key=lambda i: -abs(err[i]))[: m + 1]
        xs = np.sort(grid[pts])
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = fit()
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 100001)
    p = c32[0] + g * (c32[1] + g * (c32[2] + g * c32[3]))
    print("coefficients c0..c3 (fp32):", [float.hex(float(v)) for v in c32], [repr(float(v)) for v in c32])
    print("max relative error (exact arithmetic): %.3e" % e)
    print("max relative error (fp32 coefficients): %.3e" % np.abs(p / 2.0 ** g - 1).max())
