"""The softmax's software 2^x (soft_exp2 in csrc/ptx.cuh): the coefficients in the
source, evaluated step by step in float32 exactly as the device code does, stay
within a relative error of 1e-4 of 2^x over the range the softmax uses (the result is
then rounded to bf16, whose own rounding is 2^-9 = 1.95e-3).  CPU only."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "vision_transformer_encoder_vit_b200", "csrc",
                   "ptx.cuh")


def _coeffs():
    text = open(SRC).read()
    return [np.float32(float(re.search(rf"#define VT_EXP2_C{i} ([0-9.eE+-]+)f", text).group(1))) for i in range(4)]


def _soft_exp2(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)  # the device uses fused multiply-adds; float32 steps bound them
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    ni = t.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (ni << 23)).view(np.float32)


def test_soft_exp2_relative_error():
    x = np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32)
    got = _soft_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) < 1e-4


def test_soft_exp2_exact_at_small_integers_and_underflow():
    x = np.arange(-20, 9, dtype=np.float32)
    np.testing.assert_allclose(_soft_exp2(x), np.exp2(x.astype(np.float64)), rtol=1e-4)
    tiny = _soft_exp2(np.array([-np.inf, -1e30, -300.0, -127.0], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 1e-37)
