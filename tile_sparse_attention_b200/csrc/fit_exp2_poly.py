"""Fits the cubic used by the attention kernel's FMA-pipe exp2.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody-Waite
style range reduction; the split is exact in fp32).  2^f is approximated by a
cubic p(f) that minimises the maximum relative error |p(f) / 2^f - 1| on
[-1/2, 1/2], found with Lawson's iteratively reweighted least squares (which
converges to the minimax / Chebyshev solution).  Prints the coefficients and
the maximum relative error.

    python tile_sparse_attention_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(degree: int = 3, points: int = 20001, iters: int = 400):
    f = np.cos(np.linspace(0, np.pi, points)) * 0.5      # Chebyshev-clustered nodes
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative error rows
    b = np.ones_like(f)
    w = np.full_like(f, 1.0 / points)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        r = np.abs(A @ c - b)
        w = w * r
        w /= w.sum()
    ff = np.linspace(-0.5, 0.5, 200001)
    err = np.abs(np.polyval(c[::-1], ff) / np.exp2(ff) - 1).max()
    return c, err


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}" for v in c))
    print("max relative error on [-1/2, 1/2]:", f"{err:.3e}")
    for v in c:
        print(f"    {np.float32(v).item():.9e}f")
