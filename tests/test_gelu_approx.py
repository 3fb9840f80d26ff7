"""The fc1 epilogue's GELU (csrc/mlp.cu, gelu_erf2): erf by Abramowitz & Stegun, Handbook of
Mathematical Functions, formula 7.1.26, emulated step by step in float32 with the constants read from
the kernel source, against the exact erf GELU in float64."""
import os
import re

import numpy as np
from scipy.special import erf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MLP = os.path.join(ROOT, "structured_activation_sparsity_b200", "csrc", "mlp.cu")


def _kernel_constants():
    src = open(MLP).read()
    body = src[src.index("void gelu_erf2(float& z0, float& z1)"):]
    body = body[: body.index("\n}\n")]
    nums = [float(v) for v in re.findall(r"-?\d+\.\d+(?=f)", body)]
    # each constant is written twice (one per lane of a packed pair)
    assert all(a == b for a, b in zip(nums[0::2], nums[1::2])) and len(nums) % 2 == 0
    nums = nums[0::2]
    # the literals other than the exact 0.5, +-1, 2, in source order: 1/sqrt2, p, a5, a4, a3, a2,
    # a1, -log2(e) (the kernel multiplies x^2 by it)
    c = [v for v in nums if v not in (0.5, 1.0, -1.0, 2.0)]
    c[-1] = -c[-1]
    return [np.float32(v) for v in c]


def _emulate(z, c):
    f = np.float32
    inv_sqrt2, p, a5, a4, a3, a2, a1, log2e = c
    x = np.abs(z) * inv_sqrt2
    t = f(1) / (p * x + f(1))
    poly = t * ((((a5 * t + a4) * t + a3) * t + a2) * t + a1)
    q = poly * np.exp2(-(x * x) * log2e).astype(np.float32)
    return f(0.5) * z * np.where(z >= 0, f(2) - q, q)


def test_constants_are_the_published_ones():
    c = _kernel_constants()
    assert len(c) == 8
    published = [0.70710678118654752, 0.3275911, 1.061405429, -1.453152027, 1.421413741,
                 -0.284496736, 0.254829592, 1.4426950408889634]
    assert np.allclose(np.array(c, dtype=np.float64), published, rtol=0, atol=1e-7)


def test_error_far_below_bf16_rounding():
    z = np.linspace(-12, 12, 240001).astype(np.float32)
    g = _emulate(z, _kernel_constants()).astype(np.float64)
    zd = z.astype(np.float64)
    ref = 0.5 * zd * (1 + erf(zd / np.sqrt(2)))
    err = np.abs(g - ref)
    assert err.max() < 1e-6
    big = np.abs(ref) > 1e-3
    assert (err[big] / np.abs(ref[big])).max() < 1e-3   # bf16 keeps 2^-8 relative
