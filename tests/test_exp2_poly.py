"""The kernel's FMA-pipe 2^x (exp2_poly in attn_kernel.cuh) against the mathematical 2^x (CPU).

The constants are read from the kernel source and the same float32 steps are replayed in numpy:
magic-number rounding to the nearest integer, a cubic for 2^f on [-1/2, 1/2], exponent-field add.
Over the range the softmax feeds it ([-126, 8]: the lazy rescale keeps exponents <= 8), the relative
error must stay far below the 2^-9 rounding of the bf16 probabilities it produces.
"""

import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "temporal_block_sparse_b200", "csrc", "attn_kernel.cuh")


def _constants():
    src = open(SRC).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("}")]
    nums = [float(x) for x in re.findall(r"(-?\d+\.\d+)f", body)]
    clamp, magic = nums[0], nums[1]
    c3, c2, c1, c0 = nums[3:7]
    return clamp, magic, (c0, c1, c2, c3)


def exp2_poly_f32(x):
    clamp, magic, (c0, c1, c2, c3) = _constants()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(clamp))
    t = (x + f32(magic)).astype(f32)
    f = (x - (t - f32(magic)).astype(f32)).astype(f32)
    p = (f32(c3) * f + f32(c2)).astype(f32)
    p = (p * f + f32(c1)).astype(f32)
    p = (p * f + f32(c0)).astype(f32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_packed_variant_uses_the_same_constants():
    """exp2_poly2 (two values, packed fp32x2 ops) must use exactly the scalar version's constants."""
    src = open(SRC).read()
    body = src[src.index("float2 exp2_poly2(float2 x)"):]
    body = body[:body.index("\n}")]
    nums = {float(x) for x in re.findall(r"(-?\d+\.\d+)f", body)}
    clamp, magic, c = _constants()
    assert {clamp, magic, -magic, *c} <= nums


def test_constants_parse():
    clamp, magic, c = _constants()
    assert clamp == -126.0 and magic == 12582912.0 and abs(c[0] - 1.0) < 1e-3 and abs(c[1] - np.log(2)) < 1e-3


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.random.default_rng(0).uniform(-30, 8, 1_000_000).astype(np.float32)])
    got = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 2e-4  # bf16 rounding of P is 2^-9 = 1.95e-3


def test_integer_points_and_underflow_clamp():
    x = np.arange(-120, 9, dtype=np.float32)
    got = exp2_poly_f32(x).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=1e-4)
    tiny = exp2_poly_f32(np.array([-200.0, -np.inf], dtype=np.float32))
    assert np.all(tiny < 2.0 ** -125) and np.all(tiny >= 0)
