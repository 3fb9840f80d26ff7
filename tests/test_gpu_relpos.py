"""sparsesam_attn_relpos (SAM's decomposed relative-position bias fused into the attention) against
the oracle. Same bar as the other attention outputs: max-abs 2e-2, mean-abs 2e-3. The bias products
q.R are computed on the tensor cores in fp32 and kept in fp16 (relative rounding 2^-11), below the
bf16 rounding of q and k that every score already carries; the attention sums them into the score
exactly (fp16 times a one-hot 1.0). The permutation is the oracle's."""
import numpy as np
import pytest
import torch

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L
from structured_activation_sparsity_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
f64 = synth.bf16_to_f64


def _run(B, Hg, Wg, mode, heads, d, seed, rel_scale=0.1, units=None, head_sel=None):
    g = np.random.default_rng(seed)
    geo = O.Geometry(B, Hg, Wg, mode, 14)
    lum = g.random((B, Hg, Wg)).astype(np.float32)
    perm, _ = O.stripe_sort(O.sobel_score(lum), geo)
    U, N = geo.units, geo.unit_tokens
    Hu, Wu = O.unit_grid(geo)
    q, k, v = (synth.to_bf16(g.standard_normal((U, N, heads, 64), dtype=np.float32))
               for _ in range(3))
    rh = synth.to_bf16(g.standard_normal((2 * Hu - 1, 64), dtype=np.float32) * rel_scale)
    rw = synth.to_bf16(g.standard_normal((2 * Wu - 1, 64), dtype=np.float32) * rel_scale)
    cfg = L.make_cfg(B, Hg, Wg, mode, 14, heads, 64, d)
    wsb = L.sparsesam_attn_relpos_workspace(cfg)
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    out = torch.zeros((U, N, heads, 64), dtype=torch.bfloat16, device="cuda")
    L.sparsesam_attn_relpos(cfg, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(perm).cuda(),
                            rh.cuda(), rw.cuda(), out, ws, wsb)
    torch.cuda.synchronize()
    assert L.sparsesam_device_status() == L.SS_OK
    sel = list(range(U)) if units is None else units
    hs = list(range(heads)) if head_sel is None else head_sel
    sub = O.Geometry(1, Hg, Wg, mode, 14)
    qf, kf, vf, of = f64(q), f64(k), f64(v), f64(out)
    errs, gaps = [], []
    for u in sel:                      # units and heads are independent: one at a time
        for h in hs:
            a = [t[[u]][:, :, [h]] for t in (qf, kf, vf)]
            ref = O.attention_relpos(*a, perm[[u]], d, sub, f64(rh), f64(rw))
            errs.append(np.abs(of[[u]][:, :, [h]] - ref))
            gaps.append(np.abs(O.attention(*a, perm[[u]], d) - ref).max())
    err = np.concatenate([e.ravel() for e in errs])
    print(f"max-abs {err.max():.3e} mean-abs {err.mean():.3e}")
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    # the bias matters: without it the outputs differ well beyond the tolerance
    assert max(gaps) > 10 * MAX_ABS


@pytest.mark.parametrize("B,Hg,Wg,mode,heads,d", [
    (1, 16, 16, "global", 2, 0.4),     # b = 16: partial tiles, masks
    (1, 24, 24, "global", 2, 0.3),
    (1, 64, 64, "global", 2, 0.4),     # the ViT-B global geometry (b = 64, 16 x 16 blocks)
    (2, 20, 18, "window", 2, 0.5),     # windows of 14 x 14 with pads
])
def test_attn_relpos_matches_oracle(B, Hg, Wg, mode, heads, d):
    _run(B, Hg, Wg, mode, heads, d, seed=Hg * 3 + B)


def test_attn_relpos_vitb_full_size_sampled_units():
    """The ViT-B windowed blocks' shapes with rel-pos (4 images, 100 windows, 12 heads): units 0,
    37 and 99 checked."""
    _run(4, 64, 64, "window", 12, 0.3, seed=5, units=[0, 37, 99])


def test_attn_relpos_vitb_global_full_size():
    """The ViT-B global block's shapes with rel-pos (12 heads, 4096 tokens): heads 0, 5, 11."""
    _run(1, 64, 64, "global", 12, 0.4, seed=6, head_sel=[0, 5, 11])
