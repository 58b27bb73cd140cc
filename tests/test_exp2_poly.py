"""The prefill kernel's FMA-pipe 2^x (exp2_poly_x2 in csrc/prefill.cu), replayed
in binary32 on the CPU with the same operations in the same order, against
numpy's 2^x in binary64: relative error below 1e-4 over the range the
softmax uses (x <= 8 after the lazy rescale, down to where the clamp at -125
takes over), exact powers of two at integers, and +0-like output (2^-125) for
-inf.  The coefficients are read from the kernel source, so the test follows
any change to them."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_decode_04_b200", "csrc", "prefill.cu")


def _coefficients():
    body = open(SRC).read()
    body = body[body.index("exp2_poly_x2(uint64_t x2)"):]
    body = body[:body.index("return f32x2_pack(__int_as_float(r0)")]
    c = [float(v) for v in re.findall(r"f32x2_pack\(([0-9.]+)f, \1f\)", body)]
    assert len(c) == 4, c
    c3, c2, c1, c0 = c  # Horner order in the source: ((c3 f + c2) f + c1) f + c0
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def poly_exp2(x):
    """binary32 replay: clamp, round-to-integer by 1.5*2^23, Horner, exponent add.
    (The kernel's fma rounds once where numpy rounds twice; the bound has room.)"""
    c0, c1, c2, c3 = _coefficients()
    f32 = np.float32
    x = np.maximum(x.astype(np.float32), f32(-125.0))
    k = f32(12582912.0)
    t = (x + k).astype(np.float32)
    j = (t - k).astype(np.float32)
    f = (x - j).astype(np.float32)
    q = (f * c3 + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = (t.view(np.uint32).astype(np.uint64) << np.uint64(23)) + q.view(np.uint32).astype(np.uint64)
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-124.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()
    assert (got > 0).all()


def test_integers_and_clamp():
    for n in range(-124, 9):
        got = float(poly_exp2(np.array([n], dtype=np.float32))[0])
        assert abs(got / 2.0 ** n - 1) < 1e-4, (n, got)
    tiny = poly_exp2(np.array([-np.inf, -1e30, -125.0, -200.0], dtype=np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 3e-38)  # 2^-125: no negative or wrapped exponent
