"""Fit the polynomial of the exact-GELU kernels' complementary error function.

The kernels take erfc(w), w >= 0, in the form used by Press et al.
(Numerical Recipes, the Chebyshev-fitted "erfcc"):

    erfc(w) = t * exp(-w^2 + P(t)),   t = 1 / (1 + w / 2),

with P a polynomial in t on [0, 1] (t -> 0 as w -> infinity, where the
exact P tends to -ln(sqrt(pi)) + ln(1/2), so P is smooth on the whole
interval).  This script computes the exact P(t) = ln(erfc(w) / t) + w^2 with
mpmath at 50 digits on Chebyshev nodes of [0, 1], fits a degree-N polynomial
by least squares in the Chebyshev basis, rounds the monomial coefficients to
fp32 and reports the largest error of P (an absolute error in the exponent,
i.e. the relative error of erfc) on a dense grid, evaluated in double
arithmetic.  Run it to reproduce the constants in csrc/fk_gelu.cuh:

    python memory_bound_fk_b200/fit_erfc.py [degree]
"""
from __future__ import annotations

import sys

import mpmath
import numpy as np


def exact_p(t: float) -> float:
    if t == 0.0:
        return float(-mpmath.log(mpmath.sqrt(mpmath.pi)) + mpmath.log(mpmath.mpf(1) / 2))
    w = 2 * (1 / mpmath.mpf(t) - 1)
    return float(mpmath.log(mpmath.erfc(w) / t) + w * w)


def fit(degree: int):
    mpmath.mp.dps = 50
    n = 8 * (degree + 1)
    nodes = 0.5 - 0.5 * np.cos(np.pi * (np.arange(n) + 0.5) / n)  # Chebyshev nodes on [0, 1]
    vals = np.array([exact_p(float(t)) for t in nodes])
    cheb = np.polynomial.chebyshev.Chebyshev.fit(nodes, vals, degree, domain=[0.0, 1.0])
    mono = cheb.convert(kind=np.polynomial.Polynomial, domain=[-1, 1], window=[-1, 1]).coef
    coeffs = np.array(mono, np.float32)
    grid = np.linspace(0.0, 1.0, 4001)
    ref = np.array([exact_p(float(t)) for t in grid])
    got = np.polynomial.polynomial.polyval(grid, coeffs.astype(np.float64))
    return coeffs, float(np.max(np.abs(got - ref)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 9
    c, err = fit(deg)
    print(f"degree {deg}: max |P error| = {err:.3e} (relative error of erfc)")
    for i, v in enumerate(c):
        print(f"  c{i} = {float(v):.9e}f")
