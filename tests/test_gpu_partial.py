"""sparsesam_attn_partial (prefix + patch tokens, 2-D RoPE fused into the gather) against the oracle.

Same bar as the other attention outputs: max-abs 2e-2 and mean-abs 2e-3 (bf16 operands, fp32
accumulation and softmax). The rotation runs in fp32 on the GPU and its result is rounded to bf16
before the products, which adds at most one bf16 rounding of q and k (as any bf16 q and k carry).
The permutation is the oracle's, from the synthetic luminance of the patch grid."""
import numpy as np
import pytest
import torch

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L
from structured_activation_sparsity_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
f64 = synth.bf16_to_f64


def _run(U, Hg, Wg, prefix, heads, dh, d, base, seed, images=None):
    g = np.random.default_rng(seed)
    T = Hg * Wg
    lum = g.random((U, Hg, Wg)).astype(np.float32)
    perm, _ = O.stripe_sort(O.sobel_score(lum), O.Geometry(U, Hg, Wg, "global", 14))
    q, k, v = (synth.to_bf16(g.standard_normal((U, prefix + T, heads, dh), dtype=np.float32))
               for _ in range(3))
    cfg = L.make_cfg(U, Hg, Wg, "global", 14, heads, dh, d)
    wsb = L.sparsesam_attn_partial_workspace(cfg, prefix)
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    out = torch.zeros((U, prefix + T, heads, dh), dtype=torch.bfloat16, device="cuda")
    L.sparsesam_attn_partial(cfg, prefix, base, q.cuda(), k.cuda(), v.cuda(),
                             torch.from_numpy(perm).cuda(), out, ws, wsb)
    torch.cuda.synchronize()
    assert L.sparsesam_device_status() == L.SS_OK
    sel = list(range(U)) if images is None else images
    ref = O.attention_partial(f64(q)[sel], f64(k)[sel], f64(v)[sel], perm[sel], d, prefix, Hg, Wg,
                              base)
    err = np.abs(f64(out)[sel] - ref)
    print(f"max-abs {err.max():.3e} mean-abs {err.mean():.3e}")
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    return err


@pytest.mark.parametrize("U,Hg,Wg,prefix,heads,dh,d,base", [
    (2, 24, 24, 1, 4, 64, 0.5, 10000.0),     # PE-Core-L14-336's patch grid, one class token
    (1, 16, 16, 2, 2, 80, 0.4, 100.0),       # head dim 80, two prefix tokens
    (2, 8, 8, 0, 2, 64, 0.4, 10000.0),       # no prefix: RoPE only
    (1, 24, 24, 1, 2, 64, 0.3, 0.0),         # prefix only, no rotation
    (1, 40, 40, 1, 2, 64, 0.4, 10000.0),     # 1600 patches: the pair kernel (not short items)
])
def test_attn_partial_matches_oracle(U, Hg, Wg, prefix, heads, dh, d, base):
    _run(U, Hg, Wg, prefix, heads, dh, d, base, seed=Hg + prefix + heads)


def test_attn_partial_pe_core_l_full_size_sampled_images():
    """PE-Core-L14-336 shapes: 32 images of 1 class token + 24 x 24 patches, 16 heads x 64; the
    oracle checks images 5 and 30."""
    _run(32, 24, 24, 1, 16, 64, 0.5, 10000.0, seed=9, images=[5, 30])
