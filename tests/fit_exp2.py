"""Coefficients of the cubic used by the attention softmax to evaluate part of
its exponentials on the FMA pipe instead of the special-function unit.

2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2]; 2^f is replaced
by the cubic c0 + c1 f + c2 f^2 + c3 f^3 that minimises the maximum relative
error on [-1/2, 1/2] (Remez exchange on the relative error, started from
Chebyshev nodes).  The result feeds a bf16 probability (8 significant bits),
so a relative error near 1e-4 is far below its rounding.

Run:  python tests/fit_exp2.py
"""
import numpy as np


def remez_relative(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    for _ in range(iters):
        f = np.exp2(x)
        # c0..c_deg and the levelled error E:  p(x_i) - f_i = (-1)^i E f_i
        A = np.zeros((n, n))
        for j in range(deg + 1):
            A[:, j] = x ** j
        A[:, deg + 1] = -((-1.0) ** k) * f
        sol = np.linalg.solve(A, f)
        c = sol[: deg + 1]
        grid = np.linspace(lo, hi, 200001)
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: the extrema of the error, one per sign change region
        sign_changes = np.where(np.diff(np.sign(err)) != 0)[0]
        edges = np.concatenate([[0], sign_changes + 1, [len(grid)]])
        ext = [edges[i] + np.argmax(np.abs(err[edges[i]:edges[i + 1]])) for i in range(len(edges) - 1)]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_relative()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}" for v in c))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
