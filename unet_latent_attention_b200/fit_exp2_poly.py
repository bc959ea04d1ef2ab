"""Fits the polynomial used by the attention kernel's software exp2 (run to reproduce its constants).

The kernel evaluates part of its exponentials on the FMA pipe instead of the special-function
unit: 2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (the argument reduction of
Cody and Waite, "Software Manual for the Elementary Functions", 1980), and 2^f from a degree-3
polynomial p whose maximum relative error on [-1/2, 1/2] is minimised by the Remez exchange
algorithm (Remez, 1934). The attention probabilities are rounded to bf16 (relative step 2^-8)
right after, so the polynomial's error (about 1e-4) is far below what the result keeps.

    python -m unet_latent_attention_b200.fit_exp2_poly
"""
from __future__ import annotations

import numpy as np


def remez_rel(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    """Minimax polynomial (coefficients c0..c_deg) for 2^f on [lo, hi] in relative error."""
    n = deg + 2
    # Chebyshev extrema as the initial reference
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        f = np.exp2(x)
        # p(x_i) - f_i = (-1)^i E f_i   (weighted by f: relative error)
        A = np.hstack([x[:, None] ** np.arange(deg + 1), (-1.0) ** np.arange(n)[:, None] * f[:, None]])
        sol = np.linalg.solve(A, f)
        c = sol[:-1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = np.nonzero(np.diff(s) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.abs(err).max())


def coefficients_f32(deg: int = 3):
    c, e = remez_rel(deg)
    c32 = np.asarray(c, dtype=np.float32)
    g = np.linspace(-0.5, 0.5, 200001)
    err32 = float(np.abs((np.polyval(c32[::-1].astype(np.float64), g) - np.exp2(g)) / np.exp2(g)).max())
    return c32, e, err32


if __name__ == "__main__":
    c32, e, e32 = coefficients_f32()
    print("c0..c3 =", ", ".join(f"{float(v):.9e}f" for v in c32))
    print(f"max relative error: {e:.3e} (real coefficients), {e32:.3e} (fp32 coefficients)")
