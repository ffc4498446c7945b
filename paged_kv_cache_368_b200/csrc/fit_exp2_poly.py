"""Coefficients of the polynomial 2^f on [-1/2, 1/2] used by exp2_poly.cuh.

Method: interpolation at the Chebyshev nodes of the interval (the nodes of
T_{n+1}), which for a smooth function gives an error within a small factor
of the best (minimax) polynomial of the same degree.  The fit is computed in
float64 and the coefficients are rounded to float32, the precision the
kernel evaluates them in (Horner's rule with fused multiply-adds).

    python paged_kv_cache_368_b200/csrc/fit_exp2_poly.py     # prints the C constants

``tests/test_exp2_poly.py`` checks that the constants in exp2_poly.cuh are
what this script computes and that the float32 evaluation stays within the
error bound stated there.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def chebyshev_fit(degree: int = DEGREE) -> np.ndarray:
    """c[0..degree] with 2^f ~= sum_k c[k] f^k on [-1/2, 1/2]."""
    k = np.arange(degree + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (degree + 1)))
    vander = np.vander(nodes, degree + 1, increasing=True)
    return np.linalg.solve(vander, np.exp2(nodes))


def coefficients_f32(degree: int = DEGREE) -> np.ndarray:
    return chebyshev_fit(degree).astype(np.float32)


def horner_f32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    """The kernel's evaluation order in float32 (each step one multiply-add,
    rounded once, as fmaf does)."""
    f64 = f.astype(np.float64)
    p = np.full_like(f64, np.float64(c[-1]))
    for ck in c[-2::-1]:
        p = (p * f64 + np.float64(ck)).astype(np.float32).astype(np.float64)
    return p


def max_relative_error(degree: int = DEGREE, samples: int = 400001) -> float:
    c = coefficients_f32(degree)
    f = np.linspace(-0.5, 0.5, samples).astype(np.float32)
    return float(np.max(np.abs(horner_f32(c, f) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    for i, ck in enumerate(coefficients_f32()):
        print(f"constexpr float kExp2C{i} = {float(ck)!r}f;")
    print(f"// max relative error on [-1/2, 1/2] (float32 Horner): {max_relative_error():.3e}")
