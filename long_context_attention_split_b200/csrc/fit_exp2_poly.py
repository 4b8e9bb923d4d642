"""Fit the polynomial of exp2_poly (common.cuh): 2^f on [-0.5, 0.5],
degree 3, minimax in relative error, by the Remez exchange algorithm.

    python long_context_attention_split_b200/csrc/fit_exp2_poly.py

prints the coefficients (c0..c3, rounded to fp32) and the maximum relative
error.  exp2_poly splits x = n + f with n = round(x) (Cody and Waite's
argument reduction) and scales 2^f by 2^n through the exponent field.
"""
import numpy as np


def remez(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # c(x_i) / 2^x_i - 1 = (-1)^i E  at the n reference points
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1) / 2.0 ** x[i]
            A[i, deg + 1] = (-1) ** i
        sol = np.linalg.solve(A, np.ones(n))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1
        segs = np.split(np.arange(grid.size), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        xs = [grid[sg[np.argmax(np.abs(err[sg]))]] for sg in segs]
        if len(xs) != n:
            break
        x = np.array(xs)
    c32 = np.array(c, dtype=np.float32)
    err = np.polyval(c32.astype(np.float64)[::-1], grid) / 2.0 ** grid - 1
    return c32, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez(3)
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f")
    print(f"max relative error {e:.3e}")
