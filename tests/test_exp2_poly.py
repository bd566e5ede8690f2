"""The polynomial exp2 the kernels can use on the FMA pipe (exp2_poly2 in
fa_common.cuh): its constants are the ones gen_exp2_poly.py derives, and the
whole algorithm (round by adding 1.5 * 2^23, polynomial on [-1/2, 1/2],
integer add into the exponent field, clamp at -125), replayed in fp32 with
numpy, stays within its relative error bound of 2^x over the range the
softmax produces (x <= 8 with the lazy max, and very negative values)."""
import os
import re
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "flash_fwd_b200", "csrc")


def header_coeffs():
    src = open(os.path.join(CSRC, "fa_common.cuh")).read()
    m = re.search(r"constexpr float c0 = ([^,]+)f, c1 = ([^;]+)f;\s*constexpr float c2 = ([^,]+)f, c3 = ([^;]+)f;", src)
    assert m, "coefficients not found in fa_common.cuh"
    return np.array([float(g) for g in m.groups()], dtype=np.float32)


def test_constants_match_generator():
    sys.path.insert(0, CSRC)
    try:
        import gen_exp2_poly
    finally:
        sys.path.remove(CSRC)
    c, rel = gen_exp2_poly.fit()
    assert rel < 1e-4
    np.testing.assert_allclose(header_coeffs(), c, rtol=2e-6)


def exp2_poly_emulated(x):
    """fp32 replay of the device routine."""
    c0, c1, c2, c3 = header_coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    r = np.float32(12582912.0)
    t = (x + r).astype(np.float32)
    f = (x - (t - r)).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_range():
    x = np.linspace(-30.0, 8.0, 400001, dtype=np.float32)
    got = exp2_poly_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.abs(got / want - 1).max() < 1.5e-4


def test_underflow_is_tiny_and_positive():
    x = np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    got = exp2_poly_emulated(x)
    assert np.all(got > 0) and np.all(got < 2.0 ** -120)
