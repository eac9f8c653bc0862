"""The FMA-pipe exponential of the attention softmax (exp2_fma2 in csrc/attn_fwd.cuh).

Its arithmetic is emulated here step by step in float32 (each packed add or fma of the device
code is one float32 operation, rounded to nearest) with the coefficients read from the kernel
source, and compared with float64 exp2: the relative error over the range the softmax feeds it
(arguments from -126 to +8; the lazy rescale keeps them below 2^8) must stay far below the
bfloat16 rounding that P gets next (2^-9), and the clamp must send very negative and -inf
arguments to values no larger than 2^-126.  No GPU needed; the device code itself is covered
by the GPU parity tests when the kernels use it.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "joint_audio_video_flash_b200", "csrc", "attn_fwd.cuh")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("float2 exp2_fma2("):]
    m = re.search(r"c0 = ([0-9.e+-]+)f, c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, c3 = ([0-9.e+-]+)f",
                  body)
    assert m, "coefficients not found in exp2_fma2"
    return [np.float32(float(x)) for x in m.groups()]


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 inputs; one rounding to float32 after the add
    return (a.astype(np.float64) * b + c).astype(np.float32)


def exp2_fma_emulated(x):
    c0, c1, c2, c3 = _coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    j = (t - k).astype(np.float32)
    f = _fma32(j, np.float32(-1.0), x)
    p = _fma32(np.full_like(f, c3), f, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-126, 8, 2_000_001, dtype=np.float32),
                        np.float32([-0.5, 0.5, 0.0, -1e-7, 1e-7, 7.999, -125.5])])
    got = exp2_fma_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1.5e-4, rel.max()          # the cubic's 7.5e-5 plus float32 rounding
    assert rel.max() < 2.0 ** -9 / 10             # ten times below P's bf16 rounding


def test_integer_arguments_and_clamp():
    for e in range(-125, 9):
        v = exp2_fma_emulated(np.float32([e]))[0]
        assert abs(v / 2.0 ** e - 1) < 1e-4, e
    tiny = exp2_fma_emulated(np.float32([-126.0, -200.0, -1e30, -np.inf]))
    assert np.all(tiny >= 0) and np.all(tiny <= 2.0 ** -126 * 1.0001)
    assert np.all(np.isfinite(tiny))


def test_a_wrong_exponent_shift_or_dropped_term_is_caught():
    # the checks above would fail for plausible mistakes in the reduction
    x = np.linspace(-20, 8, 10001, dtype=np.float32)
    want = np.exp2(x.astype(np.float64))
    c0, c1, c2, c3 = _coefficients()
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    f = (x - (t - k)).astype(np.float32)
    p_no_cubic = ((c2 * f + c1) * f + c0).astype(np.float32)   # c3 dropped
    bad = (p_no_cubic.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).view(np.float32)
    assert (np.abs(bad - want) / want).max() > 1e-3
    p = ((((c3 * f + c2) * f + c1) * f) + c0).astype(np.float32)
    bad2 = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(22))).view(np.float32)
    assert (np.abs(bad2 - want) / want).max() > 1e-1
