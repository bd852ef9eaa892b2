"""Fits the polynomial the attention kernel uses to evaluate 2^f on the FMA
pipe for part of the softmax exponentials.

Method: Cody-Waite style range reduction x = n + f with n = round(x), so
f in [-1/2, 1/2], then 2^x = 2^n * p(f) where p is the degree-3 polynomial
minimising the maximum RELATIVE error on [-1/2, 1/2] (Remez exchange on the
weighted error (p - 2^f) / 2^f).  The power 2^n is applied by adding n to the
exponent field of p(f).  Run:  python fit_exp2_poly.py
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    xs = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    for _ in range(iters):
        # solve sum c_i x^i - f(x) = (-1)^j E f(x) at the reference points
        A = np.zeros((n, n))
        for j, x in enumerate(xs):
            A[j, :deg + 1] = x ** np.arange(deg + 1)
            A[j, deg + 1] = -((-1) ** j) * f(x)
        sol = np.linalg.solve(A, f(xs))
        c = sol[:deg + 1]
        grid = np.linspace(lo, hi, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: the extrema of the error between sign changes
        sign = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n:
            break
        # keep n alternating extrema with the largest magnitude
        while len(idx) > n:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        xs = grid[idx]
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez_relative()
    f32 = [float(np.float32(x)) for x in c]
    print("coefficients c0..c3 (float32):", ", ".join(f"{x!r}" for x in f32))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
