"""The FMA-pipe exponential used by the prefill softmax (csrc/exp2_fma.cuh).

Replays its float32 steps on the host with the header's coefficients (each
fused multiply-add rounded once) and checks the relative error against the
exact 2^x over the range the softmax feeds it, plus the clamp for very
negative and -inf inputs.  The end-to-end effect on the kernel is covered by
the prefill parity tests.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(__file__)), "kv_cache_decode_04_b200", "csrc",
                   "exp2_fma.cuh")


def coeffs():
    src = open(HDR).read()
    return [np.float32(float(re.search(r"#define GQA_EXP2_C%d ([0-9.eE+-]+)f" % i, src).group(1)))
            for i in range(4)]


def exp2_fma_host(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    xr = (x + magic).astype(np.float32)
    f = (x - (xr - magic).astype(np.float32)).astype(np.float32)
    fma = lambda a, b, c: (np.float64(a) * np.float64(b) + np.float64(c)).astype(np.float32)
    p = fma(c3, f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    return (p.view(np.int32) + (xr.view(np.int32) << 23)).view(np.float32)


def test_relative_error_over_softmax_range():
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = exp2_fma_host(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(got - ref) / ref).max() < 1.5e-4
    # integers are where the reduction switches n: check them and their neighbours
    xi = np.arange(-126, 9, dtype=np.float32)
    for d in (0.0, 0.4999, -0.4999, 0.5, -0.5):
        xx = (xi + np.float32(d)).astype(np.float32)
        xx = xx[(xx >= -126) & (xx <= 8)]
        rel = np.abs(exp2_fma_host(xx) - np.exp2(xx.astype(np.float64))) / np.exp2(xx.astype(np.float64))
        assert rel.max() < 1.5e-4


def test_clamp_keeps_tiny_positive_values():
    x = np.array([-126.0, -127.0, -1000.0, -np.inf], dtype=np.float32)
    y = exp2_fma_host(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 1.5e-38)
