"""Derivation of the exp2 polynomial used by the softmax warps (sm100.cuh: exp2_poly).

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody-Waite range
reduction with a single constant).  2^f is approximated by the degree-3 polynomial whose
*relative* error is minimax on [-1/2, 1/2], found here with the Remez exchange algorithm.
Run:  python fit_exp2_poly.py   (prints the float32 coefficients c0..c3 and the error bound)
"""
import numpy as np


def remez_exp2(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    n = deg + 2
    xs = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (hi - lo) / 2 + (hi + lo) / 2
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * np.exp2(x)
        c = np.linalg.solve(A, np.exp2(xs))[:deg + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        segs = np.split(np.arange(grid.size), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        new = [s[np.argmax(np.abs(err[s]))] for s in segs]
        if len(new) != n:
            break
        xs = grid[new]
    return c


if __name__ == "__main__":
    c = remez_exp2().astype(np.float32)
    g = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = ((c[3] * g + c[2]) * g + c[1]) * g + c[0]
    print("c0..c3 =", ", ".join(f"{float(x):.9g}f" for x in c))
    print("max relative error:", float(np.abs(p.astype(np.float64) / np.exp2(g.astype(np.float64)) - 1).max()))
