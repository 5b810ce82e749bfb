"""The forward kernel's FMA-pipe exponential (exp2_poly and exp2_poly_x2 in softmax_math.cuh, with
the coefficients of csrc/exp2_poly.h) emulated step by step in float32 on the CPU
and checked against 2^x: the relative error stays within the bound the header
states, over the whole range the kernel feeds it (P~ arguments up to the rescale
threshold, down to the clamp)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "exact_attention_103_b200", "csrc", "exp2_poly.h")


def _constants():
    text = open(HDR).read()
    c = [float(re.search(rf"ATTN_EXP2_C{i} ([-0-9.e]+)f", text).group(1)) for i in range(4)]
    bound = float(re.search(r"ATTN_EXP2_POLY_MAX_REL_ERR ([-0-9.e]+)", text).group(1))
    return [np.float32(x) for x in c], bound


def _fma32(a, b, c):
    """fmaf: a*b is exact in float64 for float32 a, b; one rounding to float32."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(y):
    c0, c1, c2, c3 = (np.full_like(y, c) for c in _constants()[0])
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    y = np.maximum(y, np.float32(-125.0))
    t = (y + magic).astype(np.float32)
    f = (y - (t - magic).astype(np.float32)).astype(np.float32)
    p = _fma32(f, c3, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_within_stated_bound():
    _, bound = _constants()
    y = np.linspace(-124.0, 64.0, 2_000_001).astype(np.float32)
    got = _exp2_poly(y).astype(np.float64)
    exact = np.exp2(y.astype(np.float64))
    rel = np.abs(got / exact - 1.0)
    assert rel.max() <= bound * 1.01, rel.max()


def test_integers_and_clamp():
    y = np.array([0.0, 1.0, -1.0, 8.0, -20.0, 63.0], dtype=np.float32)
    got = _exp2_poly(y).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(y.astype(np.float64)), rtol=1e-4)
    # below the clamp the result is the value at -125: tiny and positive, never a NaN
    low = _exp2_poly(np.array([-1000.0, -np.inf], dtype=np.float32))
    assert np.all(np.isfinite(low)) and np.all(low > 0) and np.all(low < 1e-37)
