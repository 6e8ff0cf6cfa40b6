"""Fits the degree-3 polynomial for 2^f on [-1/2, 1/2] used by exp2_poly_x2 (fa_device.cuh).

Remez exchange algorithm on the relative error 2^-f p(f) - 1, started from interpolation at
Chebyshev nodes; coefficients rounded to fp32.  Running it prints the coefficients (highest
degree first) and the maximum relative error of the fp32 Horner evaluation.
"""
import numpy as np


def fit(deg: int = 3, iters: int = 8):
    n = deg + 1
    x = np.cos((2 * np.arange(n) + 1) / (2 * n) * np.pi) * 0.5
    c = np.polyfit(x, 2.0 ** x, deg)
    grid = np.linspace(-0.5, 0.5, 200001)
    for _ in range(iters):
        err = np.polyval(c, grid) / 2.0 ** grid - 1
        idx = [0] + [i for i in range(1, len(grid) - 1) if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [
            len(grid) - 1]
        pts = grid[idx]
        if len(pts) != deg + 2:
            pts = np.sort(pts[np.argsort(-np.abs(err[idx]))[:deg + 2]])
        A = np.zeros((deg + 2, deg + 2))
        for r, t in enumerate(pts):
            A[r, :deg + 1] = [t ** k for k in range(deg, -1, -1)]
            A[r, deg + 1] = (-1) ** r * 2.0 ** t
        c = np.linalg.solve(A, 2.0 ** pts)[:deg + 1]
    return c.astype(np.float32)


def max_rel_error_fp32(c32) -> float:
    g = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.float32(c32[0])
    for k in c32[1:]:
        p = (p * g + k).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / 2.0 ** g.astype(np.float64) - 1).max())


if __name__ == "__main__":
    c = fit()
    print([float(v) for v in c], max_rel_error_fp32(c))
