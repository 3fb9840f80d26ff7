"""The device status word: bounded waits that run out and index checks that skip an access.

Failure is made without faulting or hanging the GPU. A wait runs out in a self-test CTA that waits,
through the kernels' own bounded-wait code, on an mbarrier nobody arrives on or a counter nobody
increments, with nothing else in flight; the wait gives up after the (shortened) limit and records
SS_ETIMEOUT. An out-of-range perm / keep entry is caught by the kernels' range checks before any
access, which record SS_EINDEX. After each, the context must still run the hot path correctly."""
import numpy as np
import pytest
import torch

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L
from structured_activation_sparsity_b200 import synth, workloads
from structured_activation_sparsity_b200.hotpath import HotPath

pytestmark = pytest.mark.gpu


def _tiny_parity():
    """One tiny block end to end, checked against the oracle (the context still works)."""
    wl = workloads.get("tiny")
    hp = HotPath(wl)
    lum = synth.luminance(wl)
    q, k, v = (synth.to_bf16(a) for a in synth.qkv(wl))
    mlp = [synth.to_bf16(a) for a in synth.mlp_params(wl, bias_scale=0.1)]
    hp.load(torch.from_numpy(lum), q, k, v, *mlp)
    hp.step()
    torch.cuda.synchronize()
    f = synth.bf16_to_f64
    geo = O.Geometry(1, 16, 16, "global", 14)
    score, perm, inv, keep, out, y = O.hot_path(lum, f(q), f(k), f(v), *(f(t) for t in mlp), geo,
                                                wl.density)
    assert np.array_equal(hp.perm.cpu().numpy(), perm)
    assert np.abs(f(hp.out) - out).max() <= 2e-2
    assert np.abs(f(hp.x) - y).max() <= 2e-2
    assert L.sparsesam_device_status() == L.SS_OK


def test_wait_that_runs_out_records_timeout_and_context_survives():
    assert L.sparsesam_device_status() == L.SS_OK
    L.sparsesam_set_wait_limit_ns(1_000_000)   # 1 ms
    try:
        for which in (0, 1):                     # mbarrier phase; global counter
            L.sparsesam_wait_selftest(which)
            assert L.sparsesam_device_status() == L.SS_ETIMEOUT, which
        for which in (2, 3):                     # the same waits, satisfied: nothing recorded
            L.sparsesam_wait_selftest(which)
            assert L.sparsesam_device_status() == L.SS_OK, which
    finally:
        L.sparsesam_set_wait_limit_ns(0)         # back to the default limit
    _tiny_parity()


def test_out_of_range_perm_and_keep_are_skipped_and_reported():
    cfg = L.make_cfg(1, 16, 16, "global", 14, 1, 64, 0.4)
    g = np.random.default_rng(3)
    lum = torch.from_numpy(g.random((1, 16, 16)).astype(np.float32)).cuda()
    score = torch.empty((1, 256), dtype=torch.float64, device="cuda")
    perm = torch.empty((1, 256), dtype=torch.int32, device="cuda")
    K = O.keep_count(0.4, 256)
    keep = torch.empty((1, K), dtype=torch.int32, device="cuda")
    L.sparsesam_score_perm(cfg, lum, score, perm, None, keep)
    q, k, v = (synth.to_bf16(g.standard_normal((1, 256, 1, 64), dtype=np.float32)).cuda()
               for _ in range(3))
    bad = perm.clone()
    bad[0, 5] = 256            # past the unit
    bad[0, 77] = -3            # negative
    out = torch.zeros_like(q)
    wsb = L.sparsesam_attn_workspace(cfg)
    ws = torch.empty((wsb,), dtype=torch.uint8, device="cuda")
    L.sparsesam_attn(cfg, q, k, v, bad, out, ws, wsb)
    assert L.sparsesam_device_status() == L.SS_EINDEX
    # keep: one entry outside the image; its row is skipped, every other row is as usual
    C, Hd = 64, 256
    x = synth.to_bf16(g.standard_normal((1, 256, C), dtype=np.float32)).cuda()
    w1 = synth.to_bf16(g.standard_normal((Hd, C), dtype=np.float32) * 0.02).cuda()
    w2 = synth.to_bf16(g.standard_normal((C, Hd), dtype=np.float32) * 0.02).cuda()
    kbad = keep.clone()
    kbad[0, 3] = 1 << 20
    x0 = x.clone()
    wsm = L.sparsesam_rcmlp_workspace(cfg, C, Hd, K)
    wm = torch.empty((wsm,), dtype=torch.uint8, device="cuda")
    L.sparsesam_rcmlp(cfg, x, C, Hd, w1, None, w2, None, kbad, K, wm, wsm)
    assert L.sparsesam_device_status() == L.SS_EINDEX
    kept = set(kbad.cpu().numpy()[0].tolist())
    untouched = [t for t in range(256) if t not in kept]
    assert torch.equal(x[0, untouched], x0[0, untouched])
    _tiny_parity()
