"""Pins of the oracle's decomposed relative-position bias (CPU only).

The bias is pinned by hand values on a 2 x 2 grid, by its defining property (for fixed q it depends
on the query/key offset only), and, with the attention, against an independent formulation: the
bias built element by element from relative-position index matrices in torch float64, added to the
scores of torch's dense attention, which the oracle must equal at density 1, for a global unit and
for padded windows."""
import math

import numpy as np
import torch

from oracle import sparsesam_oracle as O


def test_bias_hand_values_2x2():
    # Hu = Wu = 2, dh = 2: rel_h rows index qh - kh + 1, rel_w rows qw - kw + 1
    rh = np.array([[1.0, 0.0], [10.0, 0.0], [100.0, 0.0]])
    rw = np.array([[0.0, 1.0], [0.0, 20.0], [0.0, 300.0]])
    q = np.zeros((1, 4, 1, 2))
    q[0, 3, 0] = [1.0, 1.0]                  # query token (1, 1)
    b = O.relpos_bias(q, rh, rw, 2, 2)[0, 0, 3]
    # keys (0,0): rh[2] + rw[2] -> 100 + 300; (0,1): rh[2] + rw[1]; (1,0): rh[1] + rw[2]; (1,1)
    assert np.array_equal(b, [400.0, 120.0, 310.0, 30.0])


def test_bias_depends_on_offsets_only():
    g = np.random.default_rng(0)
    Hu, Wu, D = 5, 6, 8
    rh, rw = g.standard_normal((2 * Hu - 1, D)), g.standard_normal((2 * Wu - 1, D))
    qv = g.standard_normal(D)
    q = np.tile(qv, (1, Hu * Wu, 1, 1))      # the same q at every position
    b = O.relpos_bias(q, rh, rw, Hu, Wu)[0, 0]
    tok = lambda y, x: y * Wu + x
    assert b[tok(1, 1), tok(3, 4)] == b[tok(2, 2), tok(4, 5)]
    assert b[tok(4, 0), tok(1, 5)] == b[tok(3, 0), tok(0, 5)]
    assert abs(b[tok(1, 1), tok(3, 4)] - b[tok(1, 1), tok(3, 3)]) > 1e-9


def _torch_dense_relpos(q, k, v, rh, rw, Hu, Wu):
    """Dense attention with the bias built from index matrices (torch float64)."""
    qt, kt, vt = (torch.from_numpy(np.asarray(a, np.float64)).transpose(1, 2) for a in (q, k, v))
    U, H, N, D = qt.shape
    pos = torch.arange(N)
    dy = (pos // Wu)[:, None] - (pos // Wu)[None, :] + Hu - 1
    dx = (pos % Wu)[:, None] - (pos % Wu)[None, :] + Wu - 1
    Rh = torch.from_numpy(np.asarray(rh, np.float64))[dy]     # [N, N, D]
    Rw = torch.from_numpy(np.asarray(rw, np.float64))[dx]
    bias = torch.einsum("uhid,ijd->uhij", qt, Rh) + torch.einsum("uhid,ijd->uhij", qt, Rw)
    s = qt @ kt.transpose(-1, -2) / math.sqrt(D) + bias
    return (torch.softmax(s, dim=-1) @ vt).transpose(1, 2).numpy()


def test_relpos_attention_at_density_one_is_dense_global():
    g = np.random.default_rng(1)
    B, Hg, Wg, H, D = 2, 6, 8, 2, 16
    q, k, v = (g.standard_normal((B, Hg * Wg, H, D)) for _ in range(3))
    rh, rw = g.standard_normal((2 * Hg - 1, D)), g.standard_normal((2 * Wg - 1, D))
    geo = O.Geometry(B, Hg, Wg, "global", 14)
    perm = np.stack([g.permutation(Hg * Wg) for _ in range(B)]).astype(np.int32)
    y = O.attention_relpos(q, k, v, perm, 1.0, geo, rh, rw)
    ref = _torch_dense_relpos(q, k, v, rh, rw, Hg, Wg)
    assert np.allclose(y, ref, rtol=0, atol=1e-12), np.abs(y - ref).max()


def test_relpos_attention_at_density_one_is_dense_windowed():
    g = np.random.default_rng(2)
    geo = O.Geometry(1, 10, 9, "window", 4)              # 9 windows of 4 x 4 with pads
    U, N, H, D = geo.units, 16, 2, 8
    q, k, v = (g.standard_normal((U, N, H, D)) for _ in range(3))
    rh, rw = g.standard_normal((7, D)), g.standard_normal((7, D))
    perm = np.stack([g.permutation(N) for _ in range(U)]).astype(np.int32)
    y = O.attention_relpos(q, k, v, perm, 1.0, geo, rh, rw)
    ref = _torch_dense_relpos(q, k, v, rh, rw, 4, 4)
    assert np.allclose(y, ref, rtol=0, atol=1e-12)


def test_zero_tables_give_stripe_sort_attention():
    g = np.random.default_rng(3)
    lum = g.random((1, 8, 8))
    geo = O.Geometry(1, 8, 8, "global", 14)
    perm, _ = O.stripe_sort(O.sobel_score(lum), geo)
    q, k, v = (g.standard_normal((1, 64, 2, 16)) for _ in range(3))
    y = O.attention_relpos(q, k, v, perm, 0.4, geo, np.zeros((15, 16)), np.zeros((15, 16)))
    assert np.allclose(y, O.attention(q, k, v, perm, 0.4), rtol=0, atol=1e-13)
