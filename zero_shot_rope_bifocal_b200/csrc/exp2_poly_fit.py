"""Coefficients of the cubic 2^f, f in [-1/2, 1/2], used by the prefill kernel.

The kernel evaluates part of its exponentials on the FMA pipe instead of the
special-function unit: 2^x = 2^n * 2^f with n = round(x), f = x - n, and a
cubic p(f) ~ 2^f.  This script derives p: a least-squares fit of the relative
error on Chebyshev nodes, reweighted (Lawson's iteration) towards the minimax
fit.  It prints the coefficients (rounded to float32) and the maximum relative
error over a dense grid, which is 7.5e-5: below the FP16 rounding of the
probabilities (2^-11 = 4.9e-4) that the tensor core consumes.

    python zero_shot_rope_bifocal_b200/csrc/exp2_poly_fit.py
"""
import numpy as np


def fit(deg: int = 3, nodes: int = 2000, iters: int = 200):
    f = 0.5 * np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes)
    y = np.exp2(f)
    w = np.ones(nodes)
    for _ in range(iters):
        A = np.vander(f, deg + 1, increasing=True) / y[:, None]
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        err = np.abs(np.polyval(c[::-1], f) / y - 1)
        w = w * err
        w /= w.sum()
    c32 = np.float32(c)
    grid = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(np.polyval(c32[::-1].astype(np.float64), grid) / np.exp2(grid) - 1).max()
    return c32, rel


if __name__ == "__main__":
    c, rel = fit()
    print("c0..c3 =", ", ".join(f"{x:.9g}f" for x in c))
    print(f"max relative error = {rel:.3e}")
