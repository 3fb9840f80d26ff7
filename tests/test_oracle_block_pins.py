"""Pins of the oracle's full encoder block and stack (CPU only).

The block's pieces beyond S3 and S4 -- LayerNorm, the window partition with zero padding and the
crop, the qkv column order, the projections and the residual adds -- are checked against a second,
independently written formulation: SAM's ViT block as plain torch float64 library calls (layer_norm,
pad + view/permute window partition, linear, scaled_dot_product_attention, gelu). At density 1 the
Stripe-Sort pattern keeps every key, so the oracle's block must equal that dense block; a keep-set
smaller than the image must change exactly the kept rows by the MLP branch.
"""
import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import synth


def _params(C, hidden, seed, block=0):
    p = synth.block_params(C, hidden, seed, block)
    return O.BlockParams(**{k: v.astype(np.float64) for k, v in p.items()})


def _torch_block(x, prm, Hg, Wg, heads, window, keep_mask):
    """SAM's ViT block, dense attention, float64 torch; window = 0 for a global block."""
    t = lambda a: None if a is None else torch.from_numpy(np.asarray(a, np.float64))
    B, T, C = x.shape
    dh = C // heads
    xt = t(x).view(B, Hg, Wg, C)
    h = F.layer_norm(xt, (C,), t(prm.ln1_w), t(prm.ln1_b), eps=1e-6)
    if window:
        ph, pw = (-Hg) % window, (-Wg) % window
        h = F.pad(h, (0, 0, 0, pw, 0, ph))
        Hp, Wp = Hg + ph, Wg + pw
        h = h.view(B, Hp // window, window, Wp // window, window, C).permute(0, 1, 3, 2, 4, 5)
        h = h.reshape(-1, window * window, C)
    else:
        h = h.reshape(B, T, C)
    Bu, N = h.shape[:2]
    qkv = F.linear(h, t(prm.w_qkv), t(prm.b_qkv)).reshape(Bu, N, 3, heads, dh).permute(2, 0, 3, 1, 4)
    o = F.scaled_dot_product_attention(qkv[0], qkv[1], qkv[2])          # [Bu, heads, N, dh]
    o = F.linear(o.transpose(1, 2).reshape(Bu, N, C), t(prm.w_proj), t(prm.b_proj))
    if window:
        o = o.view(B, Hp // window, Wp // window, window, window, C).permute(0, 1, 3, 2, 4, 5)
        o = o.reshape(B, Hp, Wp, C)[:, :Hg, :Wg]
    x1 = xt + o.reshape(B, Hg, Wg, C)
    m = F.linear(F.gelu(F.linear(F.layer_norm(x1, (C,), t(prm.ln2_w), t(prm.ln2_b), eps=1e-6),
                                 t(prm.w1), t(prm.b1))), t(prm.w2), t(prm.b2))
    y = torch.where(torch.from_numpy(keep_mask).view(B, Hg, Wg, 1), x1 + m, x1)
    return y.reshape(B, T, C).numpy()


def test_layer_norm_hand_values():
    # [1, 2, 3, 4]: mean 5/2, variance 5/4, so (x - mean) / sqrt(5/4) = (-3, -1, 1, 3) / sqrt(5).
    y = O.layer_norm(np.array([[1.0, 2.0, 3.0, 4.0]]), np.ones(4), np.zeros(4), eps=0.0)
    assert np.allclose(y, np.array([[-3.0, -1.0, 1.0, 3.0]]) / math.sqrt(5.0), rtol=0, atol=1e-15)
    # a constant row has no deviation: the output is the bias; weight scales, bias shifts
    c = O.layer_norm(np.full((2, 6), 3.25), np.arange(6.0), np.arange(6.0) - 2.0)
    assert np.array_equal(c, np.tile(np.arange(6.0) - 2.0, (2, 1)))
    w = O.layer_norm(np.array([[1.0, 2.0, 3.0, 4.0]]), np.full(4, 2.0), np.full(4, 0.5), eps=0.0)
    assert np.allclose(w, 2.0 * y + 0.5, rtol=0, atol=1e-15)


def test_layer_norm_matches_torch():
    g = np.random.default_rng(0)
    x = g.standard_normal((5, 7, 48)) * 3 + 1
    w, b = g.standard_normal(48), g.standard_normal(48)
    ref = F.layer_norm(torch.from_numpy(x), (48,), torch.from_numpy(w), torch.from_numpy(b),
                       eps=1e-6).numpy()
    assert np.allclose(O.layer_norm(x, w, b), ref, rtol=0, atol=1e-12)


def test_units_round_trip_and_zero_pads():
    geo = O.Geometry(2, 10, 9, "window", 4)          # padded to 12 x 12: 9 windows of 16
    x = np.random.default_rng(1).standard_normal((2, 90, 3))
    u = O.to_units(x, geo)
    assert u.shape == (18, 16, 3)
    assert np.array_equal(O.from_units(u, geo), x)
    pads = sum(int((ids < 0).sum()) for _, ids in O.unit_members(geo))
    assert pads == 2 * (144 - 90)
    assert int((np.abs(u).sum(axis=2) == 0).sum()) == pads


def _check_dense(mode, Hg, Wg, window, heads, C, hidden, seed):
    B = 2
    g = np.random.default_rng(seed)
    x = g.standard_normal((B, Hg * Wg, C))
    prm = _params(C, hidden, seed)
    geo = O.Geometry(B, Hg, Wg, mode, window)
    N = geo.unit_tokens
    # any permutation: at density 1 the pattern keeps every key
    perm = np.stack([g.permutation(N) for _ in range(geo.units)]).astype(np.int32)
    keep = np.stack([g.permutation(Hg * Wg) for _ in range(B)]).astype(np.int32)
    y = O.encoder_block(x, prm, perm, keep, geo, heads, 1.0)
    ref = _torch_block(x, prm, Hg, Wg, heads, window if mode == "window" else 0,
                       np.ones((B, Hg * Wg), bool))
    assert np.allclose(y, ref, rtol=0, atol=1e-10), np.abs(y - ref).max()


def test_block_at_density_one_is_the_dense_sam_block_global():
    _check_dense("global", 8, 6, 4, 2, 32, 64, 3)


def test_block_at_density_one_is_the_dense_sam_block_windowed():
    _check_dense("window", 10, 9, 4, 2, 32, 64, 4)      # bottom/right padding in every direction


def test_block_mlp_branch_only_on_the_keep_set():
    B, Hg, Wg, C, heads = 2, 8, 8, 32, 4
    g = np.random.default_rng(5)
    x = g.standard_normal((B, Hg * Wg, C))
    prm = _params(C, 96, 5)
    geo = O.Geometry(B, Hg, Wg, "window", 4)
    perm = np.stack([np.arange(16)] * geo.units).astype(np.int32)
    keep = np.stack([g.permutation(64)[:23] for _ in range(B)]).astype(np.int32)
    mask = np.zeros((B, 64), bool)
    for b in range(B):
        mask[b, keep[b]] = True
    y = O.encoder_block(x, prm, perm, keep, geo, heads, 1.0)
    ref = _torch_block(x, prm, Hg, Wg, heads, 4, mask)
    assert np.allclose(y, ref, rtol=0, atol=1e-10)
    # the attention branch alone (no keep) leaves every row at x1: an empty keep-set
    y0 = O.encoder_block(x, prm, perm, np.zeros((B, 0), np.int32), geo, heads, 1.0)
    assert np.allclose(y0, _torch_block(x, prm, Hg, Wg, heads, 4, np.zeros((B, 64), bool)),
                       rtol=0, atol=1e-10)


def test_block_with_zero_branches_is_the_identity():
    B, Hg, Wg, C = 1, 8, 8, 32
    g = np.random.default_rng(6)
    x = g.standard_normal((B, Hg * Wg, C))
    prm = _params(C, 64, 6)
    prm.w_proj = np.zeros_like(prm.w_proj)
    prm.b_proj = None
    prm.w2 = np.zeros_like(prm.w2)
    prm.b2 = None
    geo = O.Geometry(B, Hg, Wg, "global", 4)
    perm, _ = O.stripe_sort(O.sobel_score(g.random((B, Hg, Wg))), geo)
    keep = np.arange(64, dtype=np.int32)[None, :30]
    assert np.array_equal(O.encoder_block(x, prm, perm, keep, geo, 2, 0.4), x)


def test_stack_at_density_one_is_the_dense_sam_encoder():
    B, Hg, Wg, C, heads, hidden, win = 1, 10, 10, 32, 2, 64, 4
    g = np.random.default_rng(7)
    x = g.standard_normal((B, Hg * Wg, C))
    lum = g.random((B, Hg, Wg)).astype(np.float32)
    blocks = [_params(C, hidden, 7, i) for i in range(3)]
    y = O.encoder_stack(x, blocks, lum, win, {1}, heads, 1.0)
    ref = x
    for i, prm in enumerate(blocks):
        ref = _torch_block(ref, prm, Hg, Wg, heads, 0 if i == 1 else win, np.ones((B, 100), bool))
    assert np.allclose(y, ref, rtol=0, atol=1e-9), np.abs(y - ref).max()
