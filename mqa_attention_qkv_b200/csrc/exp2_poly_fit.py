"""Fit the polynomial that the prefill softmax uses for part of its 2^x.

2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2]; 2^f is
approximated by c0 + c1 f + c2 f^2 + c3 f^3, minimax in *relative* error
(Remez exchange on the error function (p(f) - 2^f) / 2^f).  The kernel needs
P only to bf16 precision (2^-8), so degree 3 (error ~1e-4) is ample.

    python exp2_poly_fit.py        # prints the coefficients and the max error
"""
import numpy as np


def remez_rel(deg=3, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        f = np.exp2(x)
        # solve sum c_k x^k - (-1)^i E f(x_i) = f(x_i)  (relative error E)
        A = np.zeros((n, n))
        for k in range(deg + 1):
            A[:, k] = x ** k
        A[:, -1] = (-1.0) ** np.arange(n) * f
        sol = np.linalg.solve(A, f)
        c = sol[:-1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: extrema of err between sign changes
        idx = []
        sign_changes = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], sign_changes + 1, [len(grid)]])
        for a, b in zip(bounds[:-1], bounds[1:]):
            idx.append(a + np.argmax(np.abs(err[a:b])))
        idx = np.array(idx)
        if len(idx) < n:
            break
        # keep the n largest alternating extrema
        while len(idx) > n:
            drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else -1
            idx = np.delete(idx, drop)
        x = grid[idx]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_rel()
    for k, v in enumerate(c):
        print(f"c{k} = {np.float32(v)!r}  ({v:.17g})")
    print(f"max relative error {e:.3e}")
