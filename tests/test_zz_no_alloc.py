"""sparsesam_rcmlp_noalloc: the RC-MLP for callers that cannot allocate device memory (code under
another runtime's stream capture, hosts that own all device memory, loops that must avoid
cudaMalloc's device-wide synchronisation). It keeps its scratch in a fixed 32 MiB array inside the
library; its results must equal those of sparsesam_rcmlp with a caller-provided workspace.

This file is collected last so that a failure here cannot stop the rest of a -x run."""
import numpy as np
import pytest
import torch

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L
from structured_activation_sparsity_b200 import synth

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


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
    # The SAM ViT-B global block's MLP (768 -> 3072 -> 768 on 1639 kept tokens): 28 MB of scratch.
    cfg = L.make_cfg(1, 64, 64, "global", 14, 12, 64, 0.4)
    C, Hd = 768, 3072
    wsb = L.sparsesam_rcmlp_workspace(cfg, C, Hd)
    assert wsb <= 32 << 20
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    for seed in (11, 12):                                  # two calls in a row on the shared array
        x, w1, b1, w2, b2, keep = (t.to("cuda") for t in _inputs(cfg, C, Hd, seed))
        x_ref, x_new = x.clone(), x.clone()
        L.sparsesam_rcmlp(cfg, x_ref, C, Hd, w1, b1, w2, b2, keep, ws, wsb)
        L.sparsesam_rcmlp_noalloc(cfg, x_new, C, Hd, w1, b1, w2, b2, keep)
        torch.cuda.synchronize()
        err = (x_new.double() - x_ref.double()).abs()
        assert torch.isfinite(x_new.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS
        assert not torch.equal(x_new, x)                   # the kept rows did change
    assert L.sparsesam_device_status() == L.SS_OK


def test_noalloc_rejects_shapes_beyond_its_array():
    # batch 4 of the same block needs about 4 x 28 MB: rejected on the host before any CUDA call.
    cfg = L.make_cfg(4, 64, 64, "global", 14, 12, 64, 0.4)
    assert L.sparsesam_rcmlp_workspace(cfg, 768, 3072) > 32 << 20
    with pytest.raises(L.SparseSAMError) as e:
        L.sparsesam_rcmlp_noalloc(cfg, 1 << 20, 768, 3072, 1 << 20, None, 1 << 20, None, 1 << 20)
    assert e.value.code == L.SS_EWORKSPACE
