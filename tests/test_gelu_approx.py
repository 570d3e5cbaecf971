"""The normal CDF of the tensor-core TTT-MLP kernel, checked on the CPU.

The kernel evaluates GELU(x) = x Phi(x) and GELU'(x) = Phi(x) + x phi(x) with
erfc from the rational approximation of Abramowitz and Stegun, Handbook of
Mathematical Functions, formula 7.1.26 (absolute error at most 1.5e-7).  This
test reads the coefficients from the kernel source and evaluates the same
formula in float64 against scipy's erfc, so a mistyped constant fails here even
though its effect on the layer's outputs could hide under the tf32 tolerance.
"""
import os
import re

import numpy as np
from scipy.special import erfc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "test_sequence_modeling_b200", "csrc", "tc_mlp.cuh")


def coefficients():
    text = open(SRC).read()
    body = text[text.index("normal_cdf_pdf"):]
    body = body[:body.index("}")]
    vals = dict(re.findall(r"\b(P|A[1-5])\s*=\s*(-?[0-9.]+)f", body))
    assert set(vals) == {"P", "A1", "A2", "A3", "A4", "A5"}, vals
    return {k: float(v) for k, v in vals.items()}


def as_kernel_does(x, c):
    z = np.abs(x) / np.sqrt(2.0)
    t = 1.0 / (1.0 + c["P"] * z)
    poly = t * (c["A1"] + t * (c["A2"] + t * (c["A3"] + t * (c["A4"] + t * c["A5"]))))
    half_erfc = 0.5 * poly * np.exp(-0.5 * x * x)
    cdf = np.where(x >= 0, 1.0 - half_erfc, half_erfc)
    pdf = np.exp(-0.5 * x * x) / np.sqrt(2.0 * np.pi)
    return cdf, pdf


def test_erfc_within_the_published_bound():
    c = coefficients()
    z = np.linspace(0.0, 8.0, 200001)
    t = 1.0 / (1.0 + c["P"] * z)
    poly = t * (c["A1"] + t * (c["A2"] + t * (c["A3"] + t * (c["A4"] + t * c["A5"]))))
    err = np.abs(poly * np.exp(-z * z) - erfc(z))
    assert err.max() <= 1.5e-7, err.max()


def test_gelu_and_its_derivative():
    c = coefficients()
    x = np.linspace(-10.0, 10.0, 400001)
    cdf, pdf = as_kernel_does(x, c)
    exact_cdf = 0.5 * erfc(-x / np.sqrt(2.0))
    assert np.abs(cdf - exact_cdf).max() <= 7.5e-8
    # GELU and GELU' against the exact forms; GELU' by a central difference of GELU.
    gelu = x * cdf
    assert np.abs(gelu - x * exact_cdf).max() <= 7.5e-7
    h = 1e-5
    num = ((x + h) * 0.5 * erfc(-(x + h) / np.sqrt(2)) - (x - h) * 0.5 * erfc(-(x - h) / np.sqrt(2))) / (2 * h)
    assert np.abs(cdf + x * pdf - num).max() <= 1e-6
