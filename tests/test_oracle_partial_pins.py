"""Pins of the oracle's partial-token-count variant (prefix + patch tokens, 2-D RoPE), CPU only.

RoPE is pinned by closed forms (one pair at a known angle, a second frequency), by its defining
properties (a rotation keeps norms; the q.k product depends on relative positions only), and, with
the attention, against an independent formulation: channel pairs as complex numbers multiplied by
e^(i phi) in torch, then torch's dense scaled_dot_product_attention over the whole sequence, which
the oracle must equal at density 1 (every key kept)."""
import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import sparsesam_oracle as O


def test_rope_closed_form_angles():
    # dh = 4: one pair per axis at frequency base^0 = 1; token (y=1, x=2) of a 3 x 3 grid
    x = np.zeros((1, 9, 1, 4))
    x[0, 5, 0] = [1.0, 0.0, 1.0, 0.0]
    r = O.rope_2d(x, 3, 3, 100.0)[0, 5, 0]
    assert np.allclose(r, [math.cos(1), math.sin(1), math.cos(2), math.sin(2)], atol=1e-15)
    # dh = 8, base 100: pair i = 1 of each half turns at 100^(-1/2) = 0.1 per step
    x = np.zeros((1, 16, 1, 8))
    x[0, 3 * 4 + 1, 0] = [0, 0, 0.0, 1.0, 0, 0, 0.0, 1.0]      # (y=3, x=1)
    r = O.rope_2d(x, 4, 4, 100.0)[0, 13, 0]
    assert np.allclose(r[2:4], [-math.sin(0.3), math.cos(0.3)], atol=1e-15)
    assert np.allclose(r[6:8], [-math.sin(0.1), math.cos(0.1)], atol=1e-15)
    # position (0, 0) is not rotated
    z = np.random.default_rng(0).standard_normal((1, 16, 2, 8))
    assert np.array_equal(O.rope_2d(z, 4, 4, 100.0)[0, 0], z[0, 0])


def test_rope_keeps_norms_and_depends_on_relative_positions():
    g = np.random.default_rng(1)
    Hg, Wg, D = 6, 7, 16
    q = g.standard_normal((1, Hg * Wg, 1, D))
    r = O.rope_2d(q, Hg, Wg, 10000.0)
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(q, axis=-1), atol=1e-12)
    # the same q and k vectors placed at (y1, x1), (y2, x2) and then shifted by (dy, dx)
    a, b = g.standard_normal(D), g.standard_normal(D)

    def dot_at(p1, p2):
        x = np.zeros((1, Hg * Wg, 1, D))
        y = np.zeros((1, Hg * Wg, 1, D))
        x[0, p1[0] * Wg + p1[1], 0] = a
        y[0, p2[0] * Wg + p2[1], 0] = b
        ra, rb = O.rope_2d(x, Hg, Wg, 10000.0), O.rope_2d(y, Hg, Wg, 10000.0)
        return float(ra[0, p1[0] * Wg + p1[1], 0] @ rb[0, p2[0] * Wg + p2[1], 0])
    d0 = dot_at((1, 2), (3, 0))
    assert abs(dot_at((2, 4), (4, 2)) - d0) < 1e-12
    assert abs(dot_at((3, 3), (5, 1)) - d0) < 1e-12
    assert abs(dot_at((1, 3), (3, 0)) - d0) > 1e-6      # a different offset changes it


def _torch_dense(q, k, v, prefix, Hg, Wg, base):
    """Dense attention over the whole sequence with RoPE as complex rotations (torch float64)."""
    qt, kt, vt = (torch.from_numpy(np.asarray(a, np.float64)) for a in (q, k, v))
    U, NT, H, D = qt.shape
    half, quart = D // 2, D // 4
    ys = torch.arange(NT - prefix, dtype=torch.float64) // Wg
    xs = torch.arange(NT - prefix, dtype=torch.float64) % Wg
    freqs = base ** (-torch.arange(quart, dtype=torch.float64) / quart)
    ang = torch.cat([ys[:, None] * freqs[None], xs[:, None] * freqs[None]], dim=1)   # [T, D/2]
    rot = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]

    def apply(t):
        t = t.clone()
        z = torch.view_as_complex(t[:, prefix:].reshape(U, NT - prefix, H, half, 2).contiguous())
        t[:, prefix:] = torch.view_as_real(z * rot).reshape(U, NT - prefix, H, D)
        return t
    qr, kr = apply(qt), apply(kt)
    o = F.scaled_dot_product_attention(qr.transpose(1, 2), kr.transpose(1, 2), vt.transpose(1, 2))
    return o.transpose(1, 2).numpy()


def test_partial_at_density_one_is_dense_attention_with_rope():
    g = np.random.default_rng(2)
    U, Hg, Wg, H, D, prefix = 2, 6, 4, 2, 16, 1
    NT = prefix + Hg * Wg
    q, k, v = (g.standard_normal((U, NT, H, D)) for _ in range(3))
    perm = np.stack([g.permutation(Hg * Wg) for _ in range(U)]).astype(np.int32)
    y = O.attention_partial(q, k, v, perm, 1.0, prefix, Hg, Wg, 100.0)
    ref = _torch_dense(q, k, v, prefix, Hg, Wg, 100.0)
    assert np.allclose(y, ref, rtol=0, atol=1e-12), np.abs(y - ref).max()
    # two prefix tokens, no rotation
    q2, k2, v2 = (g.standard_normal((1, 2 + 16, 1, 8)) for _ in range(3))
    perm2 = g.permutation(16)[None].astype(np.int32)
    y2 = O.attention_partial(q2, k2, v2, perm2, 1.0, 2, 4, 4, 0.0)
    o2 = F.scaled_dot_product_attention(*(torch.from_numpy(a).transpose(1, 2) for a in (q2, k2, v2)))
    assert np.allclose(y2, o2.transpose(1, 2).numpy(), rtol=0, atol=1e-12)


def test_partial_without_prefix_or_rope_is_stripe_sort_attention():
    g = np.random.default_rng(3)
    lum = g.random((2, 8, 8))
    geo = O.Geometry(2, 8, 8, "global", 14)
    perm, _ = O.stripe_sort(O.sobel_score(lum), geo)
    q, k, v = (g.standard_normal((2, 64, 2, 16)) for _ in range(3))
    y = O.attention_partial(q, k, v, perm, 0.4, 0, 8, 8, 0.0)
    assert np.allclose(y, O.attention(q, k, v, perm, 0.4), rtol=0, atol=1e-13)
    # with RoPE: the same as Stripe-Sort attention of the rotated q and k
    yr = O.attention_partial(q, k, v, perm, 0.4, 0, 8, 8, 50.0)
    ref = O.attention(O.rope_2d(q, 8, 8, 50.0), O.rope_2d(k, 8, 8, 50.0), v, perm, 0.4)
    assert np.allclose(yr, ref, rtol=0, atol=1e-13)


def test_prefix_key_dominates_when_aligned():
    """A prefix key far along every patch query's direction takes (almost) all of each patch row's
    weight: the patch rows become that prefix token's value."""
    g = np.random.default_rng(4)
    U, Hg, Wg, H, D = 1, 4, 4, 1, 8
    q = np.abs(g.standard_normal((U, 17, H, D))) + 0.5
    k = g.standard_normal((U, 17, H, D)) * 0.1
    k[0, 0, 0] = 200.0                      # q . k_prefix >= 0.5 * 200 * 8 / sqrt(8) >> others
    v = g.standard_normal((U, 17, H, D))
    perm = np.arange(16, dtype=np.int32)[None]
    y = O.attention_partial(q, k, v, perm, 0.4, 1, Hg, Wg, 0.0)
    assert np.allclose(y[0, 1:, 0], np.broadcast_to(v[0, 0, 0], (16, D)), atol=1e-12)
