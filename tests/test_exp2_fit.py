"""The FMA-pipe exp2 polynomial (csrc/exp2_poly.cuh): its coefficients are the
ones paged_kv_cache_exact_b200/exp2_fit.py derives, and its relative error in
float32 stays far below half an ulp of the bf16 P it would feed."""

import os
import re

import numpy as np

from paged_kv_cache_exact_b200 import exp2_fit

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "paged_kv_cache_exact_b200", "csrc", "exp2_poly.cuh")


def _header_coefficients():
    text = open(HDR).read()
    return np.array([float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1))
                     for i in range(4)], dtype=np.float32)


def test_coefficients_match_the_fit():
    assert np.array_equal(_header_coefficients(), exp2_fit.fit())


def test_relative_error_bound():
    c = _header_coefficients()
    assert exp2_fit.max_rel_error_fp32(c) < 1e-4 < 2.0 ** -10


def test_range_reduction_reproduces_exp2():
    """The full method in float32 numpy: rint by adding 1.5*2^23, polynomial on
    the fraction, exponent added to the bits; clamp at -125."""
    c = _header_coefficients()
    x = np.linspace(-130, 8, 200001).astype(np.float32)
    xc = np.maximum(x, np.float32(-125))
    magic = np.float32(12582912.0)
    t = (xc + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (xc - r).astype(np.float32)
    p = np.full_like(f, c[3])
    for cc in c[2::-1]:
        p = (p * f + cc).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    y = bits.view(np.float32).astype(np.float64)
    want = 2.0 ** xc.astype(np.float64)
    assert np.max(np.abs(y / want - 1)) < 1e-4
    # below the clamp the result is 2^-125 up to the polynomial's error at f = 0
    assert np.all(np.abs(y[x < -125] / 2.0 ** -125 - 1) < 1e-4)
