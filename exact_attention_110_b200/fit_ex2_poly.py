"""Derives the coefficients of the cubic behind the kernels' FMA-pipe exp2 (``ex2_poly`` in
``csrc/ptx.cuh``).

The kernels split x = n + f with n = round(x) and f in [-0.5, 0.5], add n into the exponent
field, and take 2^f from a cubic c0 + c1 f + c2 f^2 + c3 f^3 evaluated in fp32 Horner form.
The cubic minimises the largest RELATIVE error |p(f) / 2^f - 1| over [-0.5, 0.5] (relative,
because the exponent addition scales the result by 2^n). Method: Lawson's algorithm, i.e.
iteratively reweighted least squares -- a weighted least-squares fit on a dense grid whose
weights are multiplied by the current absolute relative error after each solve, which drives
the fit to the minimax (equioscillating) solution. The result is rounded to fp32.

    python -m exact_attention_110_b200.fit_ex2_poly      # prints the four fp32 coefficients
"""
from __future__ import annotations

import numpy as np

GRID = 4001
ITERATIONS = 200


def fit(grid: int = GRID, iterations: int = ITERATIONS) -> np.ndarray:
    """Returns (c0, c1, c2, c3) as float32, lowest degree first."""
    f = np.linspace(-0.5, 0.5, grid)
    target = np.exp2(f)
    # Relative error p(f)/2^f - 1 is linear in the coefficients: rows are f^k / 2^f.
    A = np.stack([f ** k for k in range(4)], axis=1) / target[:, None]
    b = np.ones_like(f)
    w = np.full(grid, 1.0 / grid)
    c = np.zeros(4)
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def max_rel_error_fp32(c: np.ndarray, samples: int = 200001) -> float:
    """Largest relative error of fp32 Horner evaluation on [-0.5, 0.5] against exact 2^f."""
    f = np.linspace(-0.5, 0.5, samples).astype(np.float32)
    c = c.astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    coeffs = fit()
    for k, v in enumerate(coeffs):
        print(f"c{k} = {float(v)!r}")
    print(f"max relative error (fp32 Horner): {max_rel_error_fp32(coeffs):.3e}")
