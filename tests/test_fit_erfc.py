"""The erfc polynomial in the exact-GELU kernels is the one fit_erfc.py
produces (reproducible from the mathematics), and it meets its stated error."""
import os
import re

import numpy as np

from memory_bound_fk_b200 import fit_erfc

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "memory_bound_fk_b200", "csrc", "fk_gelu.cuh")


def test_kernel_constants_are_the_fitted_ones():
    coeffs, err = fit_erfc.fit(9)
    assert err <= 1.2e-7
    text = open(HEADER).read()
    body = text[text.index("erfc_poly(V t)"):]
    body = body[:body.index("return p;")]
    lits = [np.float32(float(v)) for v in re.findall(r"fma_v\(p, t, ([-+0-9.e]+)f\)", body)]
    first = np.float32(float(re.search(r"V p = splat_v<V>\(([-+0-9.e]+)f\);", body).group(1)))
    got = np.array([first] + lits, np.float32)[::-1]   # c0 .. c9
    assert got.shape == (10,)
    assert np.array_equal(got, coeffs)


def test_bf16_polynomial_is_the_degree_5_fit():
    """bf16 outputs take the degree-5 fit: 6.0e-5 of erfc, well under their
    half ulp (2^-9)."""
    coeffs, err = fit_erfc.fit(5)
    assert err <= 6.1e-5
    text = open(HEADER).read()
    body = text[text.index("erfc_poly5(V t)"):]
    body = body[:body.index("return p;")]
    lits = [np.float32(float(v)) for v in re.findall(r"fma_v\(p, t, ([-+0-9.e]+)f\)", body)]
    first = np.float32(float(re.search(r"V p = splat_v<V>\(([-+0-9.e]+)f\);", body).group(1)))
    got = np.array([first] + lits, np.float32)[::-1]   # c0 .. c5
    assert got.shape == (6,)
    assert np.array_equal(got, coeffs)
