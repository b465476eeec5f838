"""The cubic 2^f approximation used by exp2_fma() in the kernels (CPU check).

The coefficients compiled into sm100.cuh must be the ones the committed fit
produces (to fp32), and their fp32 Horner evaluation must stay within 8e-5
relative error on [-1/2, 1/2] -- below the 2^-9 rounding of the bf16 operands
the values feed.  The full exp2 (integer part added to the exponent field) is
checked against numpy over the range the kernels use.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.join(ROOT, "tiled_attention_16_b200", "csrc"))
import gen_exp2_poly  # noqa: E402


def header_coeffs():
    text = open(os.path.join(ROOT, "tiled_attention_16_b200", "csrc", "sm100.cuh")).read()
    body = text[text.index("float exp2_fma"):text.index("return __int_as_float")]
    nums = [float(x) for x in re.findall(r"(\d+\.\d+)f", body) if float(x) < 2.0]
    # Horner order in the source: c3, c2, c1, c0
    return np.array([nums[3], nums[2], nums[1], nums[0]], dtype=np.float32)


def exp2_fma_model(x):
    """Bit-level model of exp2_fma() in fp32."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = header_coeffs()
    p = np.full_like(f, c[3])
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_coefficients_match_fit_and_bound():
    c = header_coeffs()
    fitted = gen_exp2_poly.fit()
    np.testing.assert_allclose(c, fitted, rtol=1e-6)
    assert gen_exp2_poly.max_rel_error(c) < 8e-5


def test_full_exp2_model_against_numpy():
    x = np.concatenate([np.linspace(-120.0, 8.0, 400001), -np.logspace(-6, 2, 1001)]).astype(np.float32)
    y = exp2_fma_model(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 8e-5
    # clamp below -125: a tiny positive value, never NaN or negative
    z = exp2_fma_model(np.array([-200.0, -np.inf], dtype=np.float32))
    assert np.all(z > 0) and np.all(z < 1e-37)
