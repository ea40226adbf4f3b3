"""The FMA-pipe base-2 exponential of the tcgen05 prefill kernel, evaluated
in float32 on the host with the constants read from the kernel source: its
relative error against the exact 2^x over the range the softmax feeds it,
its exact zero for masked keys and its NaN propagation.

The kernel computes x = j + f (j the nearest integer, found by adding and
subtracting 1.5 * 2^23), p(f) = 1 + f (c1 + f (c2 + f c3)) for |f| <= 1/2,
and p(f) 2^j with 2^j built in the exponent field; x below -127 is raised to
-127, where 2^j is 0.
"""

import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "dual_flow_transformer_b200", "csrc",
                   "prefill.cu")


def _coefficients():
    text = open(SRC).read()
    c = {}
    for k in (1, 2, 3):
        m = re.search(r"constexpr float kExp2C%d = ([0-9.eE+-]+)f;" % k, text)
        assert m, "coefficient kExp2C%d not found" % k
        c[k] = np.float32(float(m.group(1)))
    return c


def _exp2_poly(x):
    c = _coefficients()
    f32 = np.float32
    x = np.asarray(x, dtype=f32)
    x = np.where(x < f32(-127), f32(-127), x).astype(f32)
    t = (x + f32(12582912.0)).astype(f32)
    j = (t - f32(12582912.0)).astype(f32)
    f = (x - j).astype(f32)
    p = (c[3] * f + c[2]).astype(f32)
    p = (p * f + c[1]).astype(f32)
    p = (p * f + f32(1)).astype(f32)
    bits = (t.view(np.int32).astype(np.int64) << 23) + 0x3F800000
    scale = (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return (p * scale).astype(f32)


def test_relative_error_over_the_softmax_range():
    # weights are 2^(s scale_log2 - m) with the reference max m at most 2^8
    # below the row's max: x in (-inf, 8]
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = _exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= 1.1e-4, rel.max()
    # far below the bf16 rounding that P then takes (2^-9 relative)
    assert rel.max() < 2.0 ** -9 / 10


def test_integers_are_exact_powers_of_two():
    x = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(_exp2_poly(x), np.exp2(x.astype(np.float64)).astype(np.float32))


def test_masked_keys_weigh_exactly_zero_and_nan_propagates():
    got = _exp2_poly(np.array([-np.inf, -1e30, -200.0, -127.0], dtype=np.float32))
    assert np.array_equal(got, np.zeros(4, dtype=np.float32))
    assert np.isnan(_exp2_poly(np.array([np.nan], dtype=np.float32))).all()
    # just above the clamp the result is tiny and non-negative (denormal range)
    tiny = _exp2_poly(np.array([-126.9, -126.5, -126.0], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny <= np.float32(2.0 ** -125))
