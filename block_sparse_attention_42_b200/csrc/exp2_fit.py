"""Fits the polynomial that the attention softmax uses to evaluate 2^f on the FMA pipe.

Method: range reduction x = n + f with n = round(x), f in [-1/2, 1/2] (Cody & Waite's
additive reduction; exact here because n is an integer), then a minimax polynomial for 2^f
on [-1/2, 1/2] found with the Remez exchange algorithm on the relative error, and 2^n
applied by adding n to the exponent field.  Prints fp32 coefficients (highest degree first)
and the fitted relative error.  Run: python exp2_fit.py [degree]
"""
import sys

import numpy as np


def remez_rel(deg, a=-0.5, b=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        grid = np.linspace(a, b, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new extrema: one per sign-alternating segment
        idx = []
        sign = np.sign(err)
        start = 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or sign[k] != sign[start]:
                seg = slice(start, k)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = k
        if len(idx) >= n:
            # keep the n largest alternating extrema
            idx = sorted(idx, key=lambda i: -abs(err[i]))[:n]
            x = np.sort(grid[idx])
    c32 = c.astype(np.float32).astype(np.float64)
    err32 = np.max(np.abs((np.polyval(c32[::-1], grid) - f(grid)) / f(grid)))
    return c.astype(np.float32), err32


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_rel(deg)
    print("coefficients c_%d .. c_0 (fp32):" % deg, ", ".join(f"{float(v):.9e}f" for v in c[::-1]))
    print(f"max relative error {e:.3e}")
