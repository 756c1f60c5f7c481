"""Error bounds of the FMA-pipe base-2 exponentials of the tcgen05 kernels.

The kernels compute 2^x as 2^f * 2^n with n = round(x) (via the 1.5 * 2^23
rounding trick), f in [-1/2, 1/2], and a fitted polynomial for 2^f: a cubic
in the forward, whose probabilities are rounded to bf16 (2^-9) anyway, and a
quartic in the scoring passes, whose sums must stay within 1e-4 of exact.
This test reads the coefficients from the CUDA header, replays the same fp32
operations in numpy and bounds the relative error against exp2.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_sparse_segment_b200", "csrc", "tc.cuh")


def coefficients(prefix="kExp2C", count=4):
    text = open(HDR).read()
    return np.float32([float(re.search(rf"{prefix}{k} = ([0-9.e+-]+)f;", text).group(1))
                       for k in range(count)])


def emulate(x, c=None):
    c = coefficients() if c is None else c
    x = np.maximum(x.astype(np.float32), np.float32(-125))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = c[-1]
    for k in range(len(c) - 2, -1, -1):   # fused multiply-add: one rounding per step
        p = (np.float64(p) * f + c[k]).astype(np.float32)
    return (p.view(np.int32) + (t.view(np.int32) << 23)).astype(np.int32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-125, 9, 1_000_001).astype(np.float32)
    rel = np.abs(emulate(x) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1e-4


def test_masked_and_exact_points():
    y = emulate(np.float32([-np.inf, 0.0, 1.0, -1.0, 8.0]))
    assert 0 < y[0] < 3e-38                      # masked logits: negligible, normal
    np.testing.assert_allclose(y[1:], [1.0, 2.0, 0.5, 256.0], rtol=1e-4)


def test_quartic_relative_error_bound():
    c = coefficients("kExp2Q", 5)
    x = np.linspace(-125, 9, 1_000_001).astype(np.float32)
    rel = np.abs(emulate(x, c) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 5e-6
    y = emulate(np.float32([-np.inf, 0.0, 3.0, -2.0]), c)
    assert 0 < y[0] < 3e-38
    np.testing.assert_allclose(y[1:], [1.0, 8.0, 0.25], rtol=5e-6)
