"""Fit of the polynomial used by ex2_poly (common.cuh): the degree-3 polynomial
p(f) ~ 2^f of least maximum relative error on [-1/2, 1/2], by the Remez
exchange algorithm.  Prints the coefficients (constant term first) rounded to
fp32 and the relative error of the fp32 Horner evaluation.

    python exact_io_aware_57_b200/csrc/ex2_poly_fit.py
"""
import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the reference points
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * 2 ** xi
        coef = np.linalg.solve(A, 2 ** x)[:deg + 1]
        err = (np.polyval(coef[::-1], grid) - 2 ** grid) / 2 ** grid
        # new reference: the extremum of each run of equal sign
        runs = [0]
        for i in range(1, len(grid)):
            if np.sign(err[i]) != np.sign(err[runs[-1]]):
                runs.append(i)
            elif abs(err[i]) > abs(err[runs[-1]]):
                runs[-1] = i
        if len(runs) >= n:
            x = grid[sorted(sorted(runs, key=lambda i: -abs(err[i]))[:n])]
    return coef


if __name__ == "__main__":
    c = remez(3).astype(np.float32)
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.zeros_like(f)
    for ci in c[::-1]:
        p = (p * f + ci).astype(np.float32)
    print("coefficients:", [float(v) for v in c])
    print("max relative error:", float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1))))
