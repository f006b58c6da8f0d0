"""Error bound of the kernels' polynomial 2^x (exp2_poly2 in csrc/sm100.cuh).

The forward softmax evaluates three of every eight pairs of exponentials on
the FMA pipe: x = j + f with j = round(x) and f in [-1/2, 1/2], 2^f by a
degree-3 polynomial, 2^j added to the exponent bits. This test replays those
steps in float32 with NumPy, using the coefficients parsed from the header,
and checks the relative error against exp2 in float64 over the whole range
the softmax feeds it (scores minus the running max, at most 2^8 above it).
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "content_adaptive_block_sa_b200", "csrc",
                   "sm100.cuh")


def _coefficients():
    src = open(HDR).read()
    got = dict(re.findall(r"kExp2C(\d) = ([0-9.eE+-]+)f", src))
    return [np.float32(float(got[str(k)])) for k in range(4)]


def _poly_exp2(x):
    c0, c1, c2, c3 = _coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    r = np.float32(12582912.0)
    t = (x + r).astype(np.float32)
    j = (t - r).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_below_bf16_rounding():
    x = np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32)
    got = _poly_exp2(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4, rel.max()  # bf16 keeps 8 bits: half an ulp is 2e-3


def test_integer_points_and_tail():
    x = np.arange(-125, 9, dtype=np.float32)
    np.testing.assert_allclose(_poly_exp2(x), np.exp2(x.astype(np.float64)), rtol=1e-4)
    # below -126 (a masked score is -inf) the result is tiny and finite, never a NaN
    tail = _poly_exp2(np.array([-126.5, -200.0, -np.inf], dtype=np.float32))
    assert np.all(np.isfinite(tail)) and np.all(tail >= 0) and np.all(tail < 2.0 ** -124)
