"""Error bound of the polynomial 2^x used for part of the softmax exponentials
in the tensor-core prefill kernel (CPU emulation of its float32 steps).

The coefficients are read from the kernel header so the test follows the code.
fmaf is emulated as a float64 multiply-add rounded once to float32 (exact here:
the float32 product is exact in float64 and the sum's rounding error is far
below float32 resolution for these magnitudes)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "chunk_wise_hierarchical_hils_b200", "csrc", "sm100.cuh")


def coeffs():
    src = open(HDR).read()
    body = src[src.index("float exp2_poly("):]
    body = body[:body.index("return")]
    nums = [float(x.rstrip("f")) for x in re.findall(r"fmaf\(fmaf\(fmaf\(fmaf\(([0-9.e-]+f), f, ([0-9.e-]+f)\), f, "
                                                     r"([0-9.e-]+f)\), f, ([0-9.e-]+f)\), f, ([0-9.e-]+f)\)", body)[0]]
    return [np.float32(x) for x in nums]   # highest degree first


def pair_coeffs():
    """Coefficients of the two-lane form, in the order they appear (highest degree first)."""
    src = open(HDR).read()
    body = src[src.index("exp2_poly_x2("):]
    body = body[body.index("const uint64_t p ="):]
    body = body[:body.index(";")]
    return [np.float32(float(x.rstrip("f"))) for x in re.findall(r"f2_splat\(([0-9.e-]+f)\)", body)]


def test_pair_form_uses_the_same_coefficients():
    assert pair_coeffs() == coeffs()


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    n = t.view(np.int32) - np.array([magic], np.float32).view(np.int32)[0]
    c4, c3, c2, c1, c0 = coeffs()
    p = fma32(fma32(fma32(fma32(np.full_like(f, c4), f, np.full_like(f, c3)), f, np.full_like(f, c2)), f,
                    np.full_like(f, c1)), f, np.full_like(f, c0))
    return (p.view(np.int32) + (n << 23)).view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 0.0, 2_000_001), -np.logspace(-8, 2, 10001), [0.0, -0.5, -1.5]])
    x = x.astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 5e-6, rel.max()


def test_clamp_and_integers():
    assert exp2_poly(np.array([0.0], np.float32))[0] == np.float32(1.0)
    assert abs(exp2_poly(np.array([-3.0], np.float32))[0] - 0.125) < 1e-9
    tiny = exp2_poly(np.array([-400.0, -126.0], np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 1e-37)
