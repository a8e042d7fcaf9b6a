"""Fit of the cubic behind the prefill kernel's FMA-pipe exponential.

The kernel (csrc/exp2_poly.cuh) computes 2^x as 2^n * p(f) with n the integer
nearest to x and f = x - n in [-1/2, 1/2]. p(f) = C0 + C1 f + C2 f^2 + C3 f^3
minimises the largest relative error |p(f) / 2^f - 1| over that interval.
This script finds it with Lawson's algorithm (C. L. Lawson, 1961): weighted
least squares on a grid, each point's weight multiplied by its current error
and renormalised after every solve, which drives the weighted solution to the
minimax one. The recipe is fixed so that it reproduces the kernel's constants
exactly: 20001 evenly spaced points on [-1/2, 1/2], uniform starting weights,
2000 iterations, coefficients rounded to float32 (round to nearest).

    python -m attention_tiled_exact_b200.exp2_poly_fit

prints the coefficients, their float32 bit patterns and the maximum relative
error of the rounded polynomial on the grid.
"""
from __future__ import annotations

import numpy as np

GRID_POINTS = 20001
ITERATIONS = 2000


def fit(grid_points: int = GRID_POINTS, iterations: int = ITERATIONS) -> np.ndarray:
    """float32 coefficients [C0, C1, C2, C3] of the minimax-relative cubic for 2^f on [-1/2, 1/2]."""
    f = np.linspace(-0.5, 0.5, grid_points)
    target = np.exp2(f)
    basis = np.vander(f, 4, increasing=True) / target[:, None]  # row i: f_i^k / 2^f_i
    w = np.full(f.size, 1.0 / f.size)
    c = None
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(basis * sw[:, None], sw, rcond=None)  # min sum w (p/2^f - 1)^2
        err = np.abs(basis @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def max_relative_error(coeffs, grid_points: int = 200001) -> float:
    """Largest |p(f) / 2^f - 1| on a dense grid, p evaluated in float64 from the float32 coefficients."""
    f = np.linspace(-0.5, 0.5, grid_points)
    c = np.asarray(coeffs, dtype=np.float64)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    return float(np.abs(p / np.exp2(f) - 1.0).max())


if __name__ == "__main__":
    c = fit()
    for i, v in enumerate(c):
        print(f"C{i} = {float(v)!r}  (0x{np.float32(v).view(np.uint32):08x})")
    print(f"max relative error on [-1/2, 1/2]: {max_relative_error(c):.4g}")
