"""Full encoder blocks and the encoder stack on the GPU against the oracle.

Each block runs through sparsesam_encoder_block (LN1 -> qkv GEMM into the permuted layout ->
attention -> proj GEMM + residual -> LN2 over the kept rows -> fc1 -> fc2 + residual) and each stack
through sparsesam_encoder_stack (one ranking of the tokens, then the blocks in order). The oracle
computes the same in float64 from the same bf16 inputs; the permutations and keep lists fed to a
single block come from the oracle too.

Tolerance. The GPU rounds to bf16 between steps (LN outputs, q/k/v, the attention output, the
MLP's hidden activation, P before P*V) and, above all, stores the residual stream x in bf16 twice
per block (after the attention branch and after the MLP branch): each store is off by up to half
an ulp, 2^-9 |x|. The bound used here is |gpu - oracle| <= n * (0.03 + 2^-7 |oracle|) for n blocks:
per block, the two residual roundings (2 * 2^-9 |x| = 2^-8 |x|, doubled for what the next steps
carry forward) plus 0.03 for the branches' own bf16 rounding. With this recipe's O(1) branches
(|x| up to about 6 after a few blocks) the worst element measured on a B200 reached 0.28 to 0.43 of
it (max-abs 0.019 to 0.025 and mean-abs about 0.002 per block)."""
import numpy as np
import pytest
import torch

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L
from structured_activation_sparsity_b200 import synth

pytestmark = pytest.mark.gpu

f64 = synth.bf16_to_f64


def _bound(ref, n_blocks):
    return n_blocks * (0.03 + 2.0 ** -7 * np.abs(ref))


def _report(y, ref, n_blocks):
    """Prints the error against the bound (pytest -s shows it) and returns the worst ratio."""
    err = np.abs(y - ref)
    r = float((err / _bound(ref, n_blocks)).max())
    print(f"max-abs {err.max():.4g} mean-abs {err.mean():.4g} worst err/bound {r:.3f}")
    return r


def _lum(B, Hg, Wg, seed):
    class _W:   # the synth luminance recipe at this grid
        batch, grid_h, grid_w = B, Hg, Wg
    return synth.luminance(_W, seed=seed)


def _weights(C, hidden, seed, block):
    """bf16 device tensors of one block (dict) and the float64 oracle parameters."""
    p = synth.block_params(C, hidden, seed, block)
    dev = {k: synth.to_bf16(v).cuda() for k, v in p.items()}
    prm = O.BlockParams(**{k: f64(t) for k, t in dev.items()})
    return dev, prm


def _block_case(B, Hg, Wg, mode, heads, dh, hidden, density, seed):
    C = heads * dh
    lum = _lum(B, Hg, Wg, seed)
    geo = O.Geometry(B, Hg, Wg, mode, 14)
    score = O.sobel_score(lum)
    perm, inv = O.stripe_sort(score, geo)
    keep = O.keep_list(score, density)
    K = keep.shape[1]
    x = synth.to_bf16(np.random.default_rng(seed).standard_normal((B, Hg * Wg, C), dtype=np.float32))
    dev, prm = _weights(C, hidden, seed, 0)
    cfg = L.make_cfg(B, Hg, Wg, mode, 14, heads, dh, density)
    wsb = L.sparsesam_encoder_block_workspace(cfg, C, hidden, K)
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    xd = x.cuda()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    L.sparsesam_encoder_block(cfg, xd, C, hidden, dev, t(perm), t(inv), t(keep), K, ws, wsb)
    torch.cuda.synchronize()
    assert L.sparsesam_device_status() == L.SS_OK
    ref = O.encoder_block(f64(x), prm, perm, keep, geo, heads, density)
    return f64(xd), ref, f64(x), keep


@pytest.mark.parametrize("B,Hg,Wg,mode,heads,dh,hidden,d", [
    (1, 16, 16, "global", 2, 64, 512, 0.4),
    (2, 20, 18, "window", 2, 64, 256, 0.5),      # padded to 28 x 28: 4 windows, pad rows dropped
    (1, 24, 24, "global", 4, 80, 640, 0.3),      # head dim 80, C = 320
    (1, 14, 30, "window", 4, 80, 384, 0.4),      # head dim 80 windows, 3 windows with pads
    (1, 32, 32, "global", 2, 64, 256, 1.0),      # dense: every key, every row through the MLP
])
def test_encoder_block_matches_oracle(B, Hg, Wg, mode, heads, dh, hidden, d):
    y, ref, x0, keep = _block_case(B, Hg, Wg, mode, heads, dh, hidden, d, seed=Hg * 7 + heads)
    _report(y, ref, 1)
    err = np.abs(y - ref)
    assert (err <= _bound(ref, 1)).all(), (err.max(), np.unravel_index(err.argmax(), err.shape))
    # both branches moved every row (the attention branch reaches every real token)
    assert (np.abs(y - x0).max(axis=2) > 0).all()


def test_encoder_block_empty_keep_set_runs_attention_branch_only():
    B, Hg, Wg, heads, dh, hidden = 1, 16, 16, 2, 64, 256
    C = heads * dh
    lum = _lum(B, Hg, Wg, 5)
    geo = O.Geometry(B, Hg, Wg, "global", 14)
    perm, inv = O.stripe_sort(O.sobel_score(lum), geo)
    x = synth.to_bf16(np.random.default_rng(5).standard_normal((B, 256, C), dtype=np.float32))
    dev, prm = _weights(C, hidden, 5, 0)
    cfg = L.make_cfg(B, Hg, Wg, "global", 14, heads, dh, 0.4)
    wsb = L.sparsesam_encoder_block_workspace(cfg, C, hidden, 0)
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    xd = x.cuda()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    L.sparsesam_encoder_block(cfg, xd, C, hidden, dev, t(perm), t(inv), None, 0, ws, wsb)
    torch.cuda.synchronize()
    ref = O.encoder_block(f64(x), prm, perm, np.zeros((B, 0), np.int32), geo, heads, 0.4)
    assert (np.abs(f64(xd) - ref) <= _bound(ref, 1)).all()


def _stack_case(B, Hg, Wg, heads, dh, hidden, density, flags, seed, images=None):
    C = heads * dh
    lum = _lum(B, Hg, Wg, seed)
    x = synth.to_bf16(np.random.default_rng(seed).standard_normal((B, Hg * Wg, C), dtype=np.float32))
    blocks = [_weights(C, hidden, seed, i) for i in range(len(flags))]
    cfg = L.make_cfg(B, Hg, Wg, "global", 14, heads, dh, density)
    wsb = L.sparsesam_encoder_stack_workspace(cfg, C, hidden)
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    xd = x.cuda()
    L.sparsesam_encoder_stack(cfg, torch.from_numpy(lum).cuda(), xd, C, hidden,
                              [b[0] for b in blocks], flags, ws, wsb)
    torch.cuda.synchronize()
    assert L.sparsesam_device_status() == L.SS_OK
    sel = list(range(B)) if images is None else images
    # images are independent: the oracle runs on the selected ones only
    ref = O.encoder_stack(f64(x)[sel], [b[1] for b in blocks], lum[sel], 14,
                          {i for i, g in enumerate(flags) if g}, heads, density)
    return f64(xd)[sel], ref


def test_encoder_stack_matches_oracle():
    flags = [False, True, False]
    y, ref = _stack_case(2, 20, 20, 2, 64, 256, 0.4, flags, seed=11)
    _report(y, ref, len(flags))
    err = np.abs(y - ref)
    assert (err <= _bound(ref, len(flags))).all(), err.max()


def test_encoder_stack_head_dim_80_matches_oracle():
    flags = [True, False]
    y, ref = _stack_case(1, 28, 28, 4, 80, 640, 0.3, flags, seed=12)
    _report(y, ref, len(flags))
    assert (np.abs(y - ref) <= _bound(ref, len(flags))).all()


def test_vitl_blocks_full_size_sampled_images():
    """The ViT-L stack's shapes (8 images of 64 x 64 tokens, C 1024 = 16 x 64, MLP 4096, density
    0.4): two windowed blocks and a global one, all 8 images on the GPU; the oracle checks images 2
    and 7 (images are independent)."""
    flags = [False, True, False]
    y, ref = _stack_case(8, 64, 64, 16, 64, 4096, 0.4, flags, seed=4, images=[2, 7])
    _report(y, ref, len(flags))
    err = np.abs(y - ref)
    assert (err <= _bound(ref, len(flags))).all(), err.max()
