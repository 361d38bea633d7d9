"""The attention kernel's polynomial 2^x (used for a quarter of the softmax
exponentials) stays within its stated error bound.

The coefficients are read from the kernel source; the range reduction and
Horner evaluation are replayed in numpy fp32 exactly as the kernel does
them (rint via the 1.5*2^23 trick, exponent added to the bits) and compared
with fp64 exp2 over the inputs the softmax feeds it (x = s*c - m <= 8).
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    src = open(os.path.join(ROOT, "kv_cache_analyzer_b200", "csrc", "attention.cu")).read()
    found = dict(re.findall(r"k(C[0-3])\s*=\s*(0x[0-9a-fA-F.p+-]+)f", src))
    return [np.float32(float.fromhex(found[f"C{i}"])) for i in range(4)]


def _exp2_poly_fp32(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    rnd = np.float32(12582912.0)
    r = (x + rnd).astype(np.float32)
    f = (x - (r - rnd)).astype(np.float32)
    p = np.float32(c3) * f
    p = (p + c2).astype(np.float32) * f          # the kernel uses fused multiply-adds;
    p = (p + c1).astype(np.float32) * f          # separate fp32 roundings here are a
    p = (p + c0).astype(np.float32)              # slightly looser replay of the same steps
    j = r.view(np.int32) - rnd.view(np.int32)
    return (p.view(np.int32) + (j << 23)).view(np.float32)


def test_reduced_range_error_bound():
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    rel = np.abs(_exp2_poly_fp32(f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
    assert rel.max() < 8e-5


def test_full_softmax_range():
    g = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125, 8, 2_000_001), g.uniform(-40, 8, 1_000_000)]).astype(np.float32)
    got = _exp2_poly_fp32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1e-4
    # integer inputs land exactly on powers of two up to the constant term
    k = np.arange(-120, 9, dtype=np.float32)
    np.testing.assert_allclose(_exp2_poly_fp32(k), np.exp2(k.astype(np.float64)), rtol=8e-5)
    # far below the clamp the result is tiny, finite and non-negative
    tiny = _exp2_poly_fp32(np.array([-1e4, -300.0, -np.inf], dtype=np.float32))
    assert np.all(np.isfinite(tiny)) and np.all(tiny >= 0) and np.all(tiny < 1e-37)
