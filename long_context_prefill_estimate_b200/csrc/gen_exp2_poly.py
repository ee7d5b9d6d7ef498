"""Coefficients of the polynomial exp2 used by the prefill kernel's softmax.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (exact in fp32 for the
x range the kernel feeds in).  2^f is approximated by the degree-3 polynomial that minimises
the maximum RELATIVE error on [-1/2, 1/2], found with a Remez exchange.  Run this file to
print the coefficients and the error bound that the kernel's constants come from:

    python long_context_prefill_estimate_b200/csrc/gen_exp2_poly.py
"""
import numpy as np


def remez_exp2(degree: int = 3, iters: int = 30):
    a, b = -0.5, 0.5
    n = degree + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i * E * 2^x_i  for the coefficients and E
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, : degree + 1] = xi ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[: degree + 1]
        grid = np.linspace(a, b, 200001)
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        idx = [0]
        for k in range(1, len(grid) - 1):
            if (err[k] - err[k - 1]) * (err[k + 1] - err[k]) <= 0:
                idx.append(k)
        idx.append(len(grid) - 1)
        idx = sorted(set(idx), key=lambda k: -abs(err[k]))[:n]
        x = np.sort(grid[idx])
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez_exp2(3)
    f32 = np.float32(c)
    grid = np.linspace(-0.5, 0.5, 100001)
    e32 = np.abs(np.polyval(f32.astype(np.float64)[::-1], grid) / 2.0 ** grid - 1).max()
    for i, ci in enumerate(f32):
        print(f"c{i} = {float(ci):.9e}f")
    print(f"max relative error: {e:.3e} (fp32 coefficients: {e32:.3e})")
