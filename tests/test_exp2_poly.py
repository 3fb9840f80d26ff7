"""The attention kernel's FMA-pipe 2^x (csrc/attn.cu, exp2_poly2), emulated step by step in float32:
its error against the exact 2^x, and its constants against their derivation (csrc/exp2_poly.py)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "structured_activation_sparsity_b200", "csrc")


def _coefficients():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m.coefficients()


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 inputs; the sum then rounds once to float32 (up to a
    # negligible double rounding) -- as the hardware fused multiply-add does.
    return _f32(np.float64(a) * np.float64(b) + np.float64(c))


def emulate(x, c):
    x = np.maximum(_f32(x), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = _f32(np.float64(x) + np.float64(magic))
    n = _f32(np.float64(t) - np.float64(magic))
    f = _fma32(n, np.float32(-1.0), x)
    q = _fma32(np.float32(c[3]), f, np.float32(c[2]))
    q = _fma32(q, f, np.float32(c[1]))
    q = _fma32(q, f, np.float32(c[0]))
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_constants_match_derivation():
    text = open(os.path.join(CSRC, "attn.cu")).read()
    body = text[text.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    lits = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    c = _coefficients()
    # Horner order in the kernel: c3 (with c2), c1, c0
    assert lits == [c[3], c[2], c[1], c[0]]


def test_relative_error_over_range():
    c = _coefficients()
    half = np.arange(-124, 8) + 0.5                      # f = +-1/2: the ends of the reduced range
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.arange(-125, 9, dtype=np.float64),
                        half, half - 1.0 + 1e-6])
    x = _f32(x[(x >= -125.0) & (x <= 8.0)])
    got = emulate(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.5e-4, rel.max()


def test_clamp_and_monotone_sign():
    c = _coefficients()
    got = emulate(np.array([-np.inf, -1e9, -200.0, -125.0], np.float32), c)
    assert np.all(got > 0) and np.all(np.isfinite(got))
    assert np.allclose(got, 2.0 ** -125, rtol=2e-4)
