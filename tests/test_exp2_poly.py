"""The FMA-pipe exp2 used for part of the softmax exponentials (CPU check of its error bound).

The kernel header states the method (round-to-nearest split x = j + f, degree-3 polynomial
for 2^f on [-1/2, 1/2], exponent add) and a maximum relative error of 7.5e-5.  This evaluates
the same float32 operations with the header's coefficients and checks that bound against
numpy's exp2, plus the clamp at -125 and exactness at integers.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "video_diffusion_attention_b200", "csrc", "sm100_ptx.cuh")


def coeffs():
    text = open(HDR).read()
    return [np.float32(float(re.search(r"kExp2C%d = ([0-9.eE+-]+)f;" % i, text).group(1)))
            for i in range(4)]


def exp2_poly(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-124.0, 8.0, 2_000_001, dtype=np.float32)
    y = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 7.6e-5
    # far below the spacing of bf16 (2^-8 relative), the type P is rounded to
    assert rel.max() < 2.0 ** -8 / 50


def test_clamp_and_signs():
    y = exp2_poly(np.array([-1e30, -200.0, -126.0, -125.0], dtype=np.float32))
    assert np.all(y > 0) and np.all(y < 3e-38)
    y = exp2_poly(np.array([float("-inf")], dtype=np.float32))
    assert 0 < y[0] < 3e-38


def test_integers_near_exact():
    x = np.arange(-120, 9, dtype=np.float32)
    y = exp2_poly(x).astype(np.float64)
    np.testing.assert_allclose(y, np.exp2(x.astype(np.float64)), rtol=7.6e-5, atol=0)
