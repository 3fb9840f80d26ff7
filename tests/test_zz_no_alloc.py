"""sparsesam_rcmlp_noalloc: the RC-MLP for callers that cannot allocate device memory at the point
where they run the block (hosts whose allocator owns all device memory, loops that must avoid
cudaMalloc's device-wide synchronisation). Its scratch is a
fixed 32 MiB array inside the library, so it takes no workspace argument.

It runs the same launches as sparsesam_rcmlp with the same plan, only over other scratch memory,
so its output must equal the workspace entry point's bit for bit. Before the compared calls, one
call with another shape leaves the shared array holding data in a different layout, which the
compared calls must not read.

This file is collected last so that a failure here cannot stop the rest of a -x run."""
import numpy as np
import pytest
import torch

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L
from structured_activation_sparsity_b200 import synth


def _inputs(cfg, C, Hd, seed):
    g = np.random.default_rng(seed)
    T = cfg.grid_h * cfg.grid_w
    lum = g.random((cfg.batch, cfg.grid_h, cfg.grid_w)).astype(np.float32)
    keep = O.keep_list(O.sobel_score(lum), cfg.density)
    x = synth.to_bf16(g.standard_normal((cfg.batch, T, C), dtype=np.float32))
    w1 = synth.to_bf16(g.standard_normal((Hd, C), dtype=np.float32) * 0.02)
    w2 = synth.to_bf16(g.standard_normal((C, Hd), dtype=np.float32) * 0.02)
    b1 = synth.to_bf16(g.standard_normal((Hd,), dtype=np.float32) * 0.1)
    b2 = synth.to_bf16(g.standard_normal((C,), dtype=np.float32) * 0.1)
    return x, w1, b1, w2, b2, torch.from_numpy(keep)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    # A different shape first (density 0.625, 512 -> 2048): it fills the array with its own layout
    # of gathered rows, hidden activations and split partials.
    cfg0 = L.make_cfg(1, 48, 48, "global", 14, 1, 64, 0.625)
    x, w1, b1, w2, b2, keep = (t.to("cuda") for t in _inputs(cfg0, 512, 2048, 7))
    L.sparsesam_rcmlp_noalloc(cfg0, x, 512, 2048, w1, b1, w2, b2, keep, keep.shape[1])
    # The SAM ViT-B global block's MLP (768 -> 3072 -> 768 on 1639 kept tokens): 28 MB of scratch.
    cfg = L.make_cfg(1, 64, 64, "global", 14, 12, 64, 0.4)
    C, Hd = 768, 3072
    K = O.keep_count(0.4, 4096)
    wsb = L.sparsesam_rcmlp_workspace(cfg, C, Hd, K)
    assert wsb <= 32 << 20
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    for seed in (11, 12):                                  # two calls in a row on the shared array
        x, w1, b1, w2, b2, keep = (t.to("cuda") for t in _inputs(cfg, C, Hd, seed))
        x_ref, x_new = x.clone(), x.clone()
        L.sparsesam_rcmlp(cfg, x_ref, C, Hd, w1, b1, w2, b2, keep, K, ws, wsb)
        L.sparsesam_rcmlp_noalloc(cfg, x_new, C, Hd, w1, b1, w2, b2, keep, K)
        torch.cuda.synchronize()
        assert torch.equal(x_new, x_ref)                   # same launches, same plan: same bits
        assert not torch.equal(x_new, x)                   # the kept rows did change
    assert L.sparsesam_device_status() == L.SS_OK


def test_noalloc_rejects_shapes_beyond_its_array():
    # batch 4 of the same block needs about 4 x 28 MB: with otherwise valid arguments it is
    # rejected on the host, before any CUDA call.
    cfg = L.make_cfg(4, 64, 64, "global", 14, 12, 64, 0.4)
    K = O.keep_count(0.4, 4096)
    assert L.sparsesam_rcmlp_workspace(cfg, 768, 3072, K) > 32 << 20
    fake = 1 << 20   # 16-byte aligned addresses that are never dereferenced
    with pytest.raises(L.SparseSAMError) as e:
        L.sparsesam_rcmlp_noalloc(cfg, fake, 768, 3072, fake, None, fake, None, fake, K)
    assert e.value.code == L.SS_EWORKSPACE
    # invalid arguments answer as sparsesam_rcmlp answers them, whatever the size
    with pytest.raises(L.SparseSAMError) as e:
        L.sparsesam_rcmlp_noalloc(cfg, None, 768, 3072, fake, None, fake, None, fake, K)
    assert e.value.code == L.SS_EINVAL
    with pytest.raises(L.SparseSAMError) as e:
        L.sparsesam_rcmlp_noalloc(cfg, fake, 760, 3072, fake, None, fake, None, fake, K)
    assert e.value.code == L.SS_EUNSUPPORTED
