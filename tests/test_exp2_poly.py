"""The cubic the softmax anchor uses for one in four of its exponentials: its
committed constants, evaluated the way the kernel does (Cody-Waite split with
the 1.5 * 2^23 rounding trick, Horner in fp32, exponent-bit add), stay within
5e-4 relative error of 2^x over the range the softmax produces, and give
exactly 0 at the clamp."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "softmax_attention_video_gated_b200", "csrc", "anchor_tc.cu")


def constants():
    src = open(SRC).read()
    vals = {k: float(v) for k, v in re.findall(r"\b(kP[123]) = ([0-9.eE+-]+)f", src)}
    return np.float32(vals["kP1"]), np.float32(vals["kP2"]), np.float32(vals["kP3"])


def fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def ex2_poly(x):
    p1, p2, p3 = constants()
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic)).astype(np.float32)
    p = fma32(fma32(fma32(np.full_like(f, p3), f, p2), f, p1), f, np.float32(1.0))
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-60.0, 8.0, 2_000_001).astype(np.float32)
    got = ex2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 5e-4, rel.max()


def test_clamp_gives_zero_and_monotone_small_values():
    x = np.array([-np.inf, -1000.0, -127.0], dtype=np.float32)
    assert np.all(ex2_poly(x) == 0.0)
    y = ex2_poly(np.array([-126.0, -100.0, -20.0], dtype=np.float32)).astype(np.float64)
    np.testing.assert_allclose(y, np.exp2([-126.0, -100.0, -20.0]), rtol=5e-4)
