"""Fit the cubic used by exp2_poly.cuh: minimax relative error of p(f) ~ 2^f on
[0, 1), by the Remez exchange algorithm.  Prints the coefficients and the
error bound; run with ``python exp2_poly_fit.py``."""
import numpy as np


def fit(deg=3, grid=200001, iters=50):
    f = np.linspace(0.0, 1.0, grid)
    target = np.exp2(f)
    n = deg + 2
    x = 0.5 - 0.5 * np.cos(np.pi * np.arange(n) / (n - 1))  # Chebyshev extrema as the start
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i: equioscillating relative error
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = (np.polyval(c[::-1], f) - target) / target
        segs = np.split(np.arange(grid), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segs]
        if len(ext) >= n:
            x = np.sort(f[sorted(ext, key=lambda i: -abs(err[i]))[:n]])
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = fit()
    print("c0..c3 =", ", ".join(f"{v:.8f}" for v in c))
    print(f"max relative error {e:.3e} (2^{np.log2(e):.2f})")
