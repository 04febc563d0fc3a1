"""The FMA-pipe exp2 of the attention kernel: constants and error bound.

The kernel computes 2^x as 2^n * p(x - n), n = round(x) obtained by adding and
subtracting 1.5 * 2^23, with a cubic p on [-1/2, 1/2].  Here the constants
compiled into the kernel are read from its source, checked against the fitting
script, and the full float32 evaluation (clamp, rounding trick, Horner steps
with fused multiply-adds emulated in float64 then rounded, the exponent-field
add of the rounded float's low bits shifted by 23) is compared with the exact
2^x over the range the kernel feeds it.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "blockwise_attn_ffn_b200", "csrc", "common.cuh")
FIT = os.path.join(ROOT, "blockwise_attn_ffn_b200", "csrc", "fit_exp2_poly.py")


def kernel_coeffs():
    s = open(SRC).read()
    return [np.float32(float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", s).group(1)))
            for i in range(4)]


def test_constants_match_fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", FIT)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    np.testing.assert_array_equal(np.array(kernel_coeffs(), np.float32), mod.fit())


def fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_kernel(x):
    c0, c1, c2, c3 = kernel_coeffs()
    magic = np.float32(12582912.0)
    x = np.maximum(np.float32(x), np.float32(-125.0)).astype(np.float32)
    j = (x + magic).astype(np.float32)
    n = (j - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = fma32(c3, f, c2)
    q = fma32(q, f, c1)
    q = fma32(q, f, c0)
    bits = (q.astype(np.float32).view(np.int32).astype(np.int64)
            + (j.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-60.0, 8.0, 400001).astype(np.float32)
    got = exp2_kernel(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.2e-4
    # far below the spacing of bfloat16 (2^-8 relative), the type P is stored in
    assert rel.max() < 2.0 ** -8 / 10


def test_large_negative_is_tiny_positive_normal():
    """The clamp keeps the exponent field positive (no wrap into the sign)."""
    for x in (-1e30, -200.0, -125.5, -125.0, -124.9):
        v = exp2_kernel(np.float32(x))
        assert 0.0 < v < 1e-37 and np.isfinite(v)
