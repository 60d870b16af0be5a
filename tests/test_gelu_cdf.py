"""The normal CDF the CUDA kernels use for the GELU MLP fast weight.

The kernels take Phi(z) from erfc(|z| / sqrt 2) by the rational approximation
of Abramowitz and Stegun, Handbook of Mathematical Functions, formula 7.1.26,
whose stated bound is |error| <= 1.5e-7 in erf. This test reads the
coefficients out of the kernel header, so it checks the numbers the device code
uses, and evaluates the formula in float64 and in float32 arithmetic over a
dense grid against math.erf. The GPU parity tests of the GELU MLP (the fp32
CUDA-core path at 1e-4) cover the device code end to end.
"""
import math
import os
import re

import numpy as np
import pytest

HDR = os.path.join(os.path.dirname(__file__), "..", "test_weight_layers_chunk_b200", "csrc",
                   "common.cuh")


def _coefficients():
    src = open(HDR).read()
    body = src[src.index("norm_cdf_pdf(float z) {"):]
    body = body[:body.index("\n}\n")]
    p = float(re.search(r"fmaf\(([-0-9.]+)f, x, 1\.0f\)", body).group(1))
    hi = re.search(r"fmaf\(t, ([-0-9.]+)f, ([-0-9.]+)f\)", body)
    rest = re.findall(r"s = fmaf\(t, s, ([-0-9.]+)f\)", body)
    a5, a4 = float(hi.group(1)), float(hi.group(2))
    a3, a2, a1 = (float(v) for v in rest)
    half_log2e = float(re.search(r"exp2f\(-([0-9.]+)f \* z \* z\)", body).group(1))
    return p, (a1, a2, a3, a4, a5), half_log2e


def _phi_as(z, dt):
    p, a, half_log2e = _coefficients()
    z = np.asarray(z, dt)
    c = lambda v: dt(v)
    e = np.exp2(-c(half_log2e) * z * z)
    x = np.abs(z) * c(1.0 / math.sqrt(2.0))
    t = c(1.0) / (c(p) * x + c(1.0))
    s = t * c(a[4]) + c(a[3])
    s = t * s + c(a[2])
    s = t * s + c(a[1])
    s = t * s + c(a[0])
    tail = c(0.5) * t * s * e
    return np.where(z >= 0, c(1.0) - tail, tail), c(1.0 / math.sqrt(2 * math.pi)) * e


def _phi_exact(z):
    return np.array([0.5 * math.erfc(-v / math.sqrt(2.0)) for v in z]), \
        np.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)


def test_constants_are_the_published_ones():
    p, a, half_log2e = _coefficients()
    assert p == pytest.approx(0.3275911, abs=0)
    assert a == pytest.approx((0.254829592, -0.284496736, 1.421413741, -1.453152027, 1.061405429),
                              abs=0)
    assert half_log2e == pytest.approx(0.5 / math.log(2.0), rel=1e-15)


def test_cdf_within_the_stated_bound_float64():
    z = np.linspace(-12.0, 12.0, 200001)
    cdf, pdf = _phi_as(z, np.float64)
    ref_cdf, ref_pdf = _phi_exact(z)
    # erf within 1.5e-7 means Phi within 0.75e-7
    assert np.max(np.abs(cdf - ref_cdf)) <= 0.75e-7
    assert np.max(np.abs(pdf - ref_pdf)) <= 1e-15
    # tail form: Phi(z) + Phi(-z) = 1 exactly in the formula's structure, but
    # at z = 0, which takes the z >= 0 side twice: Phi(0) = 1 - (a1 + ... + a5) / 2,
    # and the coefficients sum to 1 - 1e-9
    sym = np.abs(cdf + cdf[::-1] - 1.0)
    mid = len(z) // 2
    assert np.max(np.delete(sym, mid)) <= 4e-15  # rounding of 1 - tail
    assert sym[mid] <= 2e-9


def test_gelu_and_derivative_float32():
    z = np.linspace(-10.0, 10.0, 40001).astype(np.float32)
    cdf, pdf = _phi_as(z, np.float32)
    ref_cdf, ref_pdf = _phi_exact(z.astype(np.float64))
    # float32 rounding of the few operations on top of the approximation error
    assert np.max(np.abs(cdf - ref_cdf)) <= 3e-7
    z64 = z.astype(np.float64)
    g, dg = z64 * cdf, cdf + z64 * pdf
    rg, rdg = z64 * ref_cdf, ref_cdf + z64 * ref_pdf
    assert np.max(np.abs(g - rg)) <= 3e-6      # |z| <= 10
    assert np.max(np.abs(dg - rdg)) <= 1e-6
    # GELU's defining values: gelu(0) = 0, gelu'(0) = 1/2, odd part z/2
    assert g[len(z) // 2] == 0.0
    assert dg[len(z) // 2] == pytest.approx(0.5, abs=1e-7)
