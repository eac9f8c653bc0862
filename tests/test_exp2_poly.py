"""Error bound of the FMA-pipe 2^x used for part of the softmax exponentials.

The kernel's exp2_poly3 (csrc/sm100_ptx.cuh) does: clamp x at -127, n = round(x)
through the 1.5*2^23 shifter, f = x - n, degree-3 polynomial in f, then adds n<<23
to the bit pattern.  This mirrors those float32 steps in numpy and checks the
relative error against exp2 stays below 1.1e-4 (a bf16 half-ulp is 2^-9 ~ 2e-3) for
results in the normal range; below 2^-125 the result is subnormal or zero, which
contributes nothing next to a softmax row sum of at least 1.
"""
import numpy as np

C = np.array([1.0, 0.6932829022407532, 0.24221056699752808, 0.055008664727211],
             dtype=np.float32)


def exp2_poly3(x):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    n = (t - shifter).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (C[3] * f + C[2]).astype(np.float32)
    p = (p * f + C[1]).astype(np.float32)
    p = (p * f + C[0]).astype(np.float32)
    # 32-bit wrap-around add, as the integer add on the GPU (n < 0 wraps)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_poly3(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / want - 1.0)) < 1.1e-4


def test_exact_powers_and_limits():
    for k in range(-126, 9):  # exact at integers (the constant term is exactly 1)
        assert float(exp2_poly3(np.float32(k))) == 2.0 ** k
    assert float(exp2_poly3(np.float32(-np.inf))) == 0.0
    assert float(exp2_poly3(np.float32(-1000.0))) == 0.0
    assert float(exp2_poly3(np.float32(-127.0))) == 0.0
    assert 0.0 <= float(exp2_poly3(np.float32(-126.7))) < 2.0 ** -126
