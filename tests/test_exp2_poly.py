"""The FMA-pipe exponential of the softmax kernels (exp2_poly3 in csrc/common.cuh).

Its coefficients must be the ones the committed Remez fit produces, and the
kernel's fp32 steps (round-to-nearest split x = j + f with the 1.5 * 2^23
constant, Horner with fused multiply-adds, j added to the exponent field),
emulated here bit for bit in fp32, must stay within the stated relative
error of the exact 2^x over the whole range the softmax feeds it.
"""
import os
import re
import sys

import numpy as np
import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "rank_latent_attention_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly_fit  # noqa: E402

REL_BOUND = 7.5e-5  # stated in the kernel's comment


def kernel_coefficients():
    src = open(os.path.join(CSRC, "common.cuh")).read()
    body = src[src.index("float exp2_poly3(float x)"):]
    body = body[:body.index("}")]
    c3, c2 = map(float, re.search(r"fmaf\(([0-9.e-]+)f, f, ([0-9.e-]+)f\)", body).groups())
    c1 = float(re.search(r"p = fmaf\(p, f, (0\.69[0-9]+)f\)", body).group(1))
    c0 = float(re.search(r"p = fmaf\(p, f, (0\.99[0-9]+)f\)", body).group(1))
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def fma32(a, b, c):
    """fp32 fused multiply-add: the fp32 product is exact in fp64, one rounding to fp32."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly3_emulated(x, coef):
    x = np.asarray(x, dtype=np.float32)
    k = np.float32(12582912.0)
    xc = np.maximum(x, np.float32(-125.0))
    r = (xc + k).astype(np.float32)
    j = (r - k).astype(np.float32)
    f = (xc - j).astype(np.float32)
    p = fma32(np.full_like(f, coef[3]), f, np.full_like(f, coef[2]))
    p = fma32(p, f, np.full_like(f, coef[1]))
    p = fma32(p, f, np.full_like(f, coef[0]))
    bits = p.view(np.uint32) + (r.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_coefficients_are_the_remez_fit():
    coef, err = exp2_poly_fit.fit()
    assert err < REL_BOUND
    np.testing.assert_array_equal(kernel_coefficients(), coef)


def test_remez_fit_equioscillates():
    """Minimax: the weighted error of the fit reaches its bound with alternating signs n + 2 times."""
    coef = exp2_poly_fit.remez().astype(np.float64)
    f = np.linspace(-0.5, 0.5, 400001)
    e = np.polyval(coef[::-1], f) / np.exp2(f) - 1.0
    peaks = np.abs(e).max()
    # sign changes between near-extremal points
    near = e[np.abs(e) > 0.97 * peaks]
    signs = np.sign(near)
    alternations = 1 + np.count_nonzero(np.diff(signs) != 0)
    assert alternations >= 5


@pytest.mark.parametrize("lo,hi", [(-125.0, -100.0), (-100.0, -1.0), (-1.0, 1.0), (1.0, 64.0)])
def test_relative_error_bound(lo, hi):
    coef = kernel_coefficients()
    x = np.linspace(lo, hi, 1 << 18, dtype=np.float32)
    got = exp2_poly3_emulated(x, coef).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / exact - 1.0)) < REL_BOUND


def test_exact_at_integers_up_to_the_polynomial_value_at_zero():
    coef = kernel_coefficients()
    x = np.arange(-125, 65, dtype=np.float32)
    got = exp2_poly3_emulated(x, coef)
    np.testing.assert_array_equal(got, (coef[0] * np.exp2(x.astype(np.float64))).astype(np.float32))


def test_below_the_clamp_gives_a_tiny_normal():
    coef = kernel_coefficients()
    x = np.array([-125.5, -126.0, -127.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    got = exp2_poly3_emulated(x, coef)
    assert np.all(got == exp2_poly3_emulated(np.float32(-125.0), coef))
    assert np.all(got >= np.float32(1.1754944e-38))  # normal, never a denormal
    assert np.all(got < 2.36e-38)
