"""GPU parity: every hot-path step through the C ABI against the float64 oracle, on the same seeded
inputs. Score, permutation, inverse and keep list must match bit for bit; attention and RC-MLP
outputs within max-abs 2e-2 and mean-abs 2e-3 (bf16 operands, fp32 accumulation); rows outside the
keep-set bit for bit."""
import numpy as np
import pytest
import torch

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L
from structured_activation_sparsity_b200 import synth, workloads
from structured_activation_sparsity_b200.hotpath import HotPath

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
DEV = "cuda"


def _geo(cfg):
    return O.Geometry(cfg.batch, cfg.grid_h, cfg.grid_w,
                      "global" if cfg.mode == L.SS_GLOBAL else "window", cfg.window)


def _assert_close(got, want, what):
    err = np.abs(got - want)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean-abs {err.mean():.3e}"


def _status_ok():
    assert L.sparsesam_device_status() == L.SS_OK


# ------------------------------------------------------------------------------------------------
# S1 + S2: bit-exact
# ------------------------------------------------------------------------------------------------
SCORE_CASES = [
    ("tiny", None), ("vitb_global", None), ("vitb_window", None), ("vith_global", None),
]


def _score_perm(cfg, lum_np, fused=False):
    """S1 then S2 (two calls), or both through the fused call; the outputs start as NaN / -1."""
    B, H, W = lum_np.shape
    geo = _geo(cfg)
    lum = torch.from_numpy(lum_np).to(DEV)
    score = torch.full((B, H * W), float("nan"), dtype=torch.float64, device=DEV)
    perm = torch.full((geo.units, geo.unit_tokens), -1, dtype=torch.int32, device=DEV)
    inv = torch.full_like(perm, -1)
    K = O.keep_count(cfg.density, H * W)
    keep = torch.full((B, K), -1, dtype=torch.int32, device=DEV)
    if fused:
        L.sparsesam_score_perm(cfg, lum, score, perm, inv, keep)
    else:
        L.sparsesam_score(cfg, lum, score)
        L.sparsesam_perm(cfg, score, perm, inv, keep)
    torch.cuda.synchronize()
    return score.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy(), keep.cpu().numpy()


def _check_score_perm(cfg, lum_np):
    geo = _geo(cfg)
    o_score = O.sobel_score(lum_np)
    o_perm, o_inv = O.stripe_sort(o_score, geo)
    o_keep = O.keep_list(o_score, cfg.density)
    for fused in (False, True):   # both paths, bit-exact against the oracle
        score, perm, inv, keep = _score_perm(cfg, lum_np, fused)
        assert np.array_equal(score.view(np.int64), o_score.view(np.int64)), fused
        assert np.array_equal(perm, o_perm), fused
        assert np.array_equal(inv, o_inv), fused
        assert np.array_equal(keep, o_keep), fused
    _status_ok()


@pytest.mark.parametrize("name", ["tiny", "vitb_global", "vitb_window", "vith_global"])
def test_score_perm_workloads(name):
    wl = workloads.get(name)
    _check_score_perm(L.cfg_for(wl), synth.luminance(wl))


@pytest.mark.parametrize("B,H,W,mode,ws,d", [
    (1, 4, 4, "global", 14, 0.5), (2, 3, 8, "global", 14, 0.3), (1, 16, 16, "window", 6, 0.4),
    (3, 20, 28, "global", 14, 0.33), (1, 128, 128, "global", 14, 0.3), (2, 30, 30, "window", 14, 0.5),
])
def test_score_perm_edge_grids(B, H, W, mode, ws, d):
    cfg = L.make_cfg(B, H, W, mode, ws, 1, 64, d)
    g = np.random.default_rng(B * 1000 + H)
    _check_score_perm(cfg, g.random((B, H, W)).astype(np.float32))


def test_perm_ties_flat_and_quantised():
    cfg = L.make_cfg(2, 16, 16, "global", 14, 1, 64, 0.4)
    _check_score_perm(cfg, np.zeros((2, 16, 16), np.float32))          # all ties: closed form
    q = (np.random.default_rng(5).integers(0, 3, (2, 16, 16)) * 0.25).astype(np.float32)
    _check_score_perm(cfg, q)                                           # many ties
    _, perm, _, _ = _score_perm(cfg, np.full((2, 16, 16), 0.5, np.float32))
    assert np.array_equal(perm[0], [4 * k + j for j in range(4) for k in range(64)])


def _caller_scores(B, T, seed):
    """Scores a caller may pass: negatives, mixed signs, both zeros, huge and tiny magnitudes,
    infinities, subnormals and ties across signs (equal magnitudes of both signs)."""
    g = np.random.default_rng(seed)
    pool = np.array([0.0, -0.0, 1.0, -1.0, 1e308, -1e308, 1e-308, -1e-308, 5e-324, -5e-324,
                     np.inf, -np.inf, 2.5, -2.5, 3.0e-5, -3.0e-5])
    s = g.standard_normal((B, T)) * 10.0 ** g.integers(-30, 30, (B, T))
    pick = g.random((B, T)) < 0.35
    s[pick] = pool[g.integers(0, pool.size, int(pick.sum()))]
    return s


@pytest.mark.parametrize("B,H,W,mode,ws,d", [
    (2, 16, 16, "global", 14, 0.4), (1, 64, 64, "global", 14, 0.3), (2, 30, 30, "window", 14, 0.5),
    (1, 64, 64, "window", 14, 0.3),
])
def test_perm_caller_scores_any_sign(B, H, W, mode, ws, d):
    """sparsesam_perm on scores it did not compute: it must rank by value, -0.0 tying with +0.0."""
    cfg = L.make_cfg(B, H, W, mode, ws, 1, 64, d)
    geo = _geo(cfg)
    sc = _caller_scores(B, H * W, seed=B * 100 + H)
    o_perm, o_inv = O.stripe_sort(sc, geo)
    o_keep = O.keep_list(sc, cfg.density)
    dsc = torch.from_numpy(sc).to(DEV)
    perm = torch.full((geo.units, geo.unit_tokens), -1, dtype=torch.int32, device=DEV)
    inv = torch.full_like(perm, -1)
    keep = torch.full(o_keep.shape, -1, dtype=torch.int32, device=DEV)
    L.sparsesam_perm(cfg, dsc, perm, inv, keep)
    torch.cuda.synchronize()
    assert np.array_equal(perm.cpu().numpy(), o_perm)
    assert np.array_equal(inv.cpu().numpy(), o_inv)
    assert np.array_equal(keep.cpu().numpy(), o_keep)
    _status_ok()


def test_perm_negative_zero_ties_positive_zero():
    """All scores zero, half of them -0.0: one tie class, so the closed form of a flat image."""
    cfg = L.make_cfg(1, 16, 16, "global", 14, 1, 64, 0.4)
    sc = np.zeros((1, 256))
    sc[0, ::2] = -0.0
    dsc = torch.from_numpy(sc).to(DEV)
    perm = torch.empty((1, 256), dtype=torch.int32, device=DEV)
    L.sparsesam_perm(cfg, dsc, perm, None, None)
    torch.cuda.synchronize()
    assert np.array_equal(perm.cpu().numpy()[0], [4 * k + j for j in range(4) for k in range(64)])


# ------------------------------------------------------------------------------------------------
# S3 attention
# ------------------------------------------------------------------------------------------------
def _attn_case(cfg, seed, scale=1.0, heads_check=None, units_check=None):
    """heads_check / units_check: None (all) or a list of the heads / units the oracle checks."""
    geo = _geo(cfg)
    U, N, H, D = geo.units, geo.unit_tokens, cfg.heads, cfg.head_dim
    g = np.random.default_rng(seed)
    lum = g.random((cfg.batch, cfg.grid_h, cfg.grid_w)).astype(np.float32)
    qkv = [synth.to_bf16(g.standard_normal((U, N, H, D), dtype=np.float32) * scale) for _ in range(3)]
    _, perm, _, _ = _score_perm(cfg, lum)
    dq, dk, dv = (t.to(DEV) for t in qkv)
    dperm = torch.from_numpy(perm).to(DEV)
    out = torch.full_like(dq, float("nan"))
    wsb = L.sparsesam_attn_workspace(cfg)
    ws = torch.empty((wsb,), dtype=torch.uint8, device=DEV)
    L.sparsesam_attn(cfg, dq, dk, dv, dperm, out, ws, wsb)
    torch.cuda.synchronize()
    got = synth.bf16_to_f64(out)
    us = np.arange(U) if units_check is None else np.asarray(units_check)
    hs = np.arange(H) if heads_check is None else np.asarray(heads_check)
    q64, k64, v64 = (synth.bf16_to_f64(t)[us][:, :, hs] for t in qkv)
    want = O.attention(q64, k64, v64, perm[us], cfg.density)
    _assert_close(got[us][:, :, hs], want, f"attn {U}x{N}x{H}x{D} d={cfg.density}")
    _status_ok()
    return got, want


@pytest.mark.parametrize("B,H,W,mode,heads,dh,d", [
    (1, 16, 16, "global", 1, 64, 0.4),     # tiny: b=16, masked tiles, 2 query tiles
    (1, 32, 32, "global", 2, 64, 0.3),     # b=64, nb=4
    (2, 32, 32, "global", 2, 64, 1.0),     # dense
    (1, 16, 16, "global", 2, 80, 0.4),     # head_dim 80
    (1, 28, 28, "window", 2, 64, 0.3),     # 4 windows of 196 tokens: ragged tail tile
    (1, 20, 20, "window", 1, 80, 0.5),     # windows with pads, dh 80
    (4, 56, 56, "window", 4, 64, 0.4),     # 512 short items: CTAs run two or more item pairs
    (1, 4, 4, "global", 1, 64, 0.6),       # N=16, b=1
    (1, 6, 6, "global", 3, 64, 0.5),       # N=36, b=1, nb=9
    (1, 48, 48, "global", 2, 64, 0.4),     # N=2304, b=64 (L=576 -> b=64, nb=9)
])
def test_attention_small(B, H, W, mode, heads, dh, d):
    cfg = L.make_cfg(B, H, W, mode, 14, heads, dh, d)
    _attn_case(cfg, seed=H * 7 + heads)


def test_attention_tiny_workload():
    wl = workloads.get("tiny")
    _attn_case(L.cfg_for(wl), seed=0, scale=wl.qkv_scale)


# Full sizes: every unit and head of ViT-B global; elsewhere a spread sample (first, middle and
# last units; first, middle and last heads), so that an indexing slip past the first unit or head
# cannot pass.
@pytest.mark.parametrize("name,heads_check,units_check", [
    ("vitb_global", None, None), ("vitb_window", [0, 5, 11], [0, 1, 49, 50, 98, 99]),
    ("vith_global", [0, 7, 15], [0, 2, 3]), ("vitl_global", [0, 9, 15], [0, 7]),
])
def test_attention_full_size(name, heads_check, units_check):
    wl = workloads.get(name)
    _attn_case(L.cfg_for(wl), seed=wl.seed, scale=wl.qkv_scale, heads_check=heads_check,
               units_check=units_check)


# ------------------------------------------------------------------------------------------------
# S4 RC-MLP
# ------------------------------------------------------------------------------------------------
def _mlp_case(cfg, C, Hd, seed, bias=True, images_check=None):
    """images_check: None (all) or a list of the images the oracle checks (the residual rows of
    every image are checked bit for bit)."""
    B, T = cfg.batch, cfg.grid_h * cfg.grid_w
    g = np.random.default_rng(seed)
    lum = g.random((B, cfg.grid_h, cfg.grid_w)).astype(np.float32)
    _, _, _, keep = _score_perm(cfg, lum)
    x = synth.to_bf16(g.standard_normal((B, T, C), dtype=np.float32))
    w1 = synth.to_bf16(g.standard_normal((Hd, C), dtype=np.float32) * 0.02)
    w2 = synth.to_bf16(g.standard_normal((C, Hd), dtype=np.float32) * 0.02)
    b1 = synth.to_bf16(g.standard_normal((Hd,), dtype=np.float32) * 0.1) if bias else None
    b2 = synth.to_bf16(g.standard_normal((C,), dtype=np.float32) * 0.1) if bias else None
    dx = x.to(DEV)
    dev = [None if t is None else t.to(DEV) for t in (w1, b1, w2, b2)]
    dkeep = torch.from_numpy(keep).to(DEV)
    K = keep.shape[1]
    wsb = L.sparsesam_rcmlp_workspace(cfg, C, Hd, K)
    ws = torch.empty((wsb,), dtype=torch.uint8, device=DEV)
    L.sparsesam_rcmlp(cfg, dx, C, Hd, dev[0], dev[1], dev[2], dev[3], dkeep, K, ws, wsb)
    torch.cuda.synchronize()
    got = synth.bf16_to_f64(dx)
    x64 = synth.bf16_to_f64(x)
    bs = np.arange(B) if images_check is None else np.asarray(images_check)
    want = O.rcmlp(x64[bs], synth.bf16_to_f64(w1), None if b1 is None else synth.bf16_to_f64(b1),
                   synth.bf16_to_f64(w2), None if b2 is None else synth.bf16_to_f64(b2), keep[bs])
    mask = np.zeros((B, T), bool)
    for b in range(B):
        mask[b, keep[b]] = True
    assert np.array_equal(got[~mask], x64[~mask]), "residual rows changed"
    m = mask[bs]
    _assert_close(got[bs][m], want[m], f"rcmlp B={B} T={T} C={C} H={Hd}")
    _status_ok()


@pytest.mark.parametrize("B,H,W,C,Hd,d,bias", [
    (1, 16, 16, 64, 256, 0.4, True),       # tiny shape, K=103 < one M tile
    (2, 16, 16, 128, 512, 0.5, False),
    (1, 32, 32, 256, 1024, 0.3, True),
    (3, 20, 20, 192, 320, 1.0, True),      # dense, N not a multiple of 128 (BN 64)
    (1, 32, 32, 128, 2048, 0.4, True),     # fc2 split four ways along K: the last split finishes
    (1, 48, 48, 384, 1536, 0.5, True),     # fc2 split two ways, all units resident: paired finish
    (1, 64, 64, 768, 3072, 0.625, True),   # paired finish with 256-wide tiles (120 units)
    (2, 48, 48, 512, 2048, 0.5, True),     # paired finish with 128-wide tiles (144 units)
])
def test_rcmlp_small(B, H, W, C, Hd, d, bias):
    cfg = L.make_cfg(B, H, W, "global", 14, 1, 64, d)
    _mlp_case(cfg, C, Hd, seed=C + Hd, bias=bias)


@pytest.mark.parametrize("name,images_check", [("vitb_global", None), ("vitb_window", [0, 3]),
                                               ("vith_global", [0, 3]), ("vitl_global", [0, 7])])
def test_rcmlp_full_size(name, images_check):
    wl = workloads.get(name)
    _mlp_case(L.cfg_for(wl), wl.dim, wl.hidden, seed=wl.seed, images_check=images_check)


# ------------------------------------------------------------------------------------------------
# The whole block through HotPath
# ------------------------------------------------------------------------------------------------
def test_hotpath_tiny_end_to_end():
    wl = workloads.get("tiny")
    hp = HotPath(wl)
    lum = synth.luminance(wl)
    q, k, v = (synth.to_bf16(a) for a in synth.qkv(wl))
    x, w1, b1, w2, b2 = synth.mlp_params(wl, bias_scale=0.1)
    xb, w1b, b1b, w2b, b2b = (synth.to_bf16(a) for a in (x, w1, b1, w2, b2))
    hp.load(torch.from_numpy(lum), q, k, v, xb, w1b, b1b, w2b, b2b)
    n0 = L.sparsesam_launch_count()
    hp.step()
    torch.cuda.synchronize()
    assert L.sparsesam_launch_count() - n0 == 6   # S1+S2 fused, gather, attn, gather, fc1, fc2
    geo = O.Geometry(1, 16, 16, "global", 14)
    score, perm, inv, keep, out, y = O.hot_path(
        lum, *(synth.bf16_to_f64(t) for t in (q, k, v, xb, w1b, b1b, w2b, b2b)), geo, wl.density)
    assert np.array_equal(hp.score.cpu().numpy().view(np.int64), score.view(np.int64))
    assert np.array_equal(hp.perm.cpu().numpy(), perm)
    assert np.array_equal(hp.inv.cpu().numpy(), inv)
    assert np.array_equal(hp.keep.cpu().numpy(), keep)
    _assert_close(synth.bf16_to_f64(hp.out), out, "hotpath attn")
    _assert_close(synth.bf16_to_f64(hp.x), y, "hotpath rcmlp")
    _status_ok()


def test_trace_records_each_launch():
    wl = workloads.get("tiny")
    hp = HotPath(wl)
    hp.load(torch.from_numpy(synth.luminance(wl)), *(synth.to_bf16(a) for a in synth.qkv(wl)),
            *(synth.to_bf16(a) for a in synth.mlp_params(wl)))
    L.sparsesam_trace_start(64)
    hp.step()
    recs = L.sparsesam_trace_stop()
    names = [n for n, _ in recs]
    assert names == ["score_rank", "gather_qkv", "attn", "gather_rows", "rcmlp_fc1", "rcmlp_fc2"]
    assert all(ms > 0 for _, ms in recs)


# ------------------------------------------------------------------------------------------------
# The whole-block call against the per-step calls: the same kernels on the same data, so every
# output is bit-identical.
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny", "vitb_global", "vitb_window", "vith_global"])
def test_block_call_equals_step_calls(name):
    wl = workloads.get(name)
    a, b = HotPath(wl), HotPath(wl)
    lum = torch.from_numpy(synth.luminance(wl))
    q, k, v = (synth.to_bf16(t) for t in synth.qkv(wl))
    mlp = [synth.to_bf16(t) for t in synth.mlp_params(wl, bias_scale=0.1)]
    a.load(lum, q, k, v, *mlp)
    b.load(lum, q, k, v, *mlp)
    a.step()
    b.step_by_calls()
    torch.cuda.synchronize()
    for ta, tb in ((a.score, b.score), (a.perm, b.perm), (a.inv, b.inv), (a.keep, b.keep),
                   (a.out, b.out), (a.x, b.x)):
        assert torch.equal(ta.view(torch.int8) if ta.dtype != torch.int32 else ta,
                           tb.view(torch.int8) if tb.dtype != torch.int32 else tb), name
    _status_ok()
