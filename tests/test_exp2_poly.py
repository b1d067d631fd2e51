"""The software 2^x of the tensor-core kernel, checked on the CPU.

The kernel computes a share of the softmax exponentials with a cubic on the FMA
pipe (fb_tc_kernel.cuh, exp2_poly2).  This test reads the coefficients from the
kernel source, replays the same fp32 steps with numpy (round-to-nearest shifter,
cubic, exponent-field add) and checks the relative error against 2^x, far below
the bf16 rounding (2^-9) that P gets afterwards."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "cached_split_attention_b200", "csrc", "fb_tc_kernel.cuh")


def _coefficients():
    text = open(SRC).read()
    c = {}
    for i in range(4):
        m = re.search(rf"constexpr float kExpC{i} = ([0-9.eE+-]+)f;", text)
        assert m, f"kExpC{i} not found"
        c[i] = np.float32(float(m.group(1)))
    return c


def _exp2_poly(x):
    c = _coefficients()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    shift = f32(12582912.0)
    t = (x + shift).astype(f32)
    f = (x - (t - shift).astype(f32)).astype(f32)
    q = (c[3] * f + c[2]).astype(f32)  # the kernel fuses these multiply-adds; the
    q = (q * f + c[1]).astype(f32)     # unfused fp32 steps here round a little more
    q = (q * f + c[0]).astype(f32)
    bits = q.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-120.0, 8.0, 400001, dtype=np.float32)  # lazily rescaled scores stay <= 8
    got = _exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.5e-4, rel.max()


def test_masked_scores_give_nothing():
    x = np.array([-np.inf, -1e30, -200.0, -126.0], dtype=np.float32)
    got = _exp2_poly(x)
    assert np.all(got >= 0.0) and np.all(got < 2.0 ** -125)


def test_integers_are_nearly_exact():
    x = np.arange(-100, 9, dtype=np.float32)
    rel = np.abs(_exp2_poly(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4
