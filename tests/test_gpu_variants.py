"""GPU parity of the variants: the random-permutation ablation (the README's `sparsesam_random`)
and the keep-set by update magnitude (Dutch summary, "Selectieve Berekening"), each through the C ABI
against the float64 oracle. Scores, permutations, magnitudes and keep lists bit for bit; the RC-MLP
on an update-magnitude keep-set within max-abs 2e-2 / mean-abs 2e-3."""
import numpy as np
import pytest
import torch

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L
from structured_activation_sparsity_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("B,H,W,mode,ws,d,seed", [
    (1, 16, 16, "global", 14, 0.4, 0), (2, 64, 64, "global", 14, 0.3, 12345),
    (2, 64, 64, "window", 14, 0.3, 7), (3, 20, 28, "global", 14, 0.5, 2**63 + 5),
])
def test_random_perm_matches_oracle(B, H, W, mode, ws, d, seed):
    cfg = L.make_cfg(B, H, W, mode, ws, 1, 64, d)
    geo = O.Geometry(B, H, W, mode, ws)
    o_sc = O.random_scores(B, H * W, seed)
    o_perm, o_inv = O.stripe_sort(o_sc, geo)
    o_keep = O.keep_list(o_sc, d)
    sc = torch.full((B, H * W), float("nan"), dtype=torch.float64, device=DEV)
    perm = torch.full((geo.units, geo.unit_tokens), -1, dtype=torch.int32, device=DEV)
    inv = torch.full_like(perm, -1)
    keep = torch.full(o_keep.shape, -1, dtype=torch.int32, device=DEV)
    L.sparsesam_random_perm(cfg, seed, sc, perm, inv, keep)
    torch.cuda.synchronize()
    assert np.array_equal(sc.cpu().numpy().view(np.int64), o_sc.view(np.int64))
    assert np.array_equal(perm.cpu().numpy(), o_perm)
    assert np.array_equal(inv.cpu().numpy(), o_inv)
    assert np.array_equal(keep.cpu().numpy(), o_keep)
    assert L.sparsesam_device_status() == L.SS_OK


def _delta(B, T, C, seed, ties=False):
    g = np.random.default_rng(seed)
    d = g.standard_normal((B, T, C), dtype=np.float32) * g.uniform(0.1, 3.0, size=(B, T, 1)).astype(np.float32)
    if ties:
        d[:, ::7] = 0.0                  # many zero magnitudes
        d[:, 1::5] = d[:, 3:4]           # many equal rows
    return synth.to_bf16(d)


@pytest.mark.parametrize("B,H,W,C,K,ties", [
    (1, 16, 16, 64, 103, False), (2, 64, 64, 768, 1229, True), (4, 64, 64, 1280, 1229, False),
    (1, 8, 8, 16, 0, False), (1, 8, 8, 16, 64, True), (2, 12, 12, 1024, 17, True),
])
def test_keep_by_update_matches_oracle(B, H, W, C, K, ties):
    cfg = L.make_cfg(B, H, W, "global", 14, 1, 64, 0.5)
    T = H * W
    delta = _delta(B, T, C, seed=C + K, ties=ties)
    o_mag = O.update_magnitude(synth.bf16_to_f64(delta))
    o_keep = O.keep_top(o_mag, K)
    mag = torch.full((B, T), float("nan"), dtype=torch.float64, device=DEV)
    keep = torch.full((B, max(K, 1)), -1, dtype=torch.int32, device=DEV)
    L.sparsesam_keep_by_update(cfg, delta.to(DEV), C, K, mag, keep)
    torch.cuda.synchronize()
    if K:
        assert np.array_equal(mag.cpu().numpy().view(np.int64), o_mag.view(np.int64))
        assert np.array_equal(keep.cpu().numpy()[:, :K], o_keep)
    else:   # K = 0: nothing launched, nothing written
        assert torch.isnan(mag).all() and (keep == -1).all()
    assert L.sparsesam_device_status() == L.SS_OK


def test_rcmlp_on_update_magnitude_keep_set():
    """The variant end to end: keep-set by update magnitude, then the RC-MLP on it."""
    B, H, W, C, Hd, K = 2, 32, 32, 256, 1024, 300
    cfg = L.make_cfg(B, H, W, "global", 14, 1, 64, 0.4)
    T = H * W
    g = np.random.default_rng(9)
    delta = _delta(B, T, C, seed=3)
    x = synth.to_bf16(g.standard_normal((B, T, C), dtype=np.float32))
    w1 = synth.to_bf16(g.standard_normal((Hd, C), dtype=np.float32) * 0.02)
    w2 = synth.to_bf16(g.standard_normal((C, Hd), dtype=np.float32) * 0.02)
    b1 = synth.to_bf16(g.standard_normal((Hd,), dtype=np.float32) * 0.1)
    b2 = synth.to_bf16(g.standard_normal((C,), dtype=np.float32) * 0.1)
    mag = torch.empty((B, T), dtype=torch.float64, device=DEV)
    keep = torch.empty((B, K), dtype=torch.int32, device=DEV)
    L.sparsesam_keep_by_update(cfg, delta.to(DEV), C, K, mag, keep)
    dx = x.to(DEV)
    wsb = L.sparsesam_rcmlp_workspace(cfg, C, Hd, K)
    ws = torch.empty((wsb,), dtype=torch.uint8, device=DEV)
    L.sparsesam_rcmlp(cfg, dx, C, Hd, w1.to(DEV), b1.to(DEV), w2.to(DEV), b2.to(DEV), keep, K, ws, wsb)
    torch.cuda.synchronize()
    o_keep = O.keep_top(O.update_magnitude(synth.bf16_to_f64(delta)), K)
    assert np.array_equal(keep.cpu().numpy(), o_keep)
    f = synth.bf16_to_f64
    want = O.rcmlp(f(x), f(w1), f(b1), f(w2), f(b2), o_keep)
    got = f(dx)
    mask = np.zeros((B, T), bool)
    for b in range(B):
        mask[b, o_keep[b]] = True
    assert np.array_equal(got[~mask], f(x)[~mask])
    err = np.abs(got[mask] - want[mask])
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert L.sparsesam_device_status() == L.SS_OK
