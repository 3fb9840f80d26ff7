"""CPU checks of the C-ABI library: it loads, exports every declared symbol, validates arguments on
the host before touching a GPU, and its static pattern equals the oracle's bit for bit."""
import ctypes
import math
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import sparsesam_oracle as O
from structured_activation_sparsity_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparsesam.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*[a-z_0-9 ]+\*?\s*\**\s*(sparsesam_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L.lib, n)


def test_no_launches_without_gpu_work():
    assert L.sparsesam_launch_count() == 0


def test_strerror():
    assert L.strerror(0) == "ok"
    for c in (-1, -2, -3, -4, -5, -6):
        assert L.strerror(c) != "unknown error"
    assert L.strerror(-99) == "unknown error"


# ---- pattern / blocklist equal the oracle ----------------------------------------------------
CASES = [
    (1, 16, 16, "global", 0.4), (1, 64, 64, "global", 0.4), (4, 64, 64, "global", 0.3),
    (1, 64, 64, "global", 0.5), (1, 64, 64, "global", 1.0), (2, 64, 64, "window", 0.3),
    (2, 64, 64, "window", 0.4), (2, 64, 64, "window", 0.5), (1, 32, 32, "global", 0.25),
    (1, 8, 8, "global", 0.5), (1, 4, 4, "global", 0.6), (1, 6, 6, "global", 0.5),
    (1, 16, 16, "window", 0.7), (1, 20, 28, "global", 0.33), (3, 128, 128, "global", 0.3),
]


@pytest.mark.parametrize("B,H,W,mode,d", CASES)
def test_pattern_matches_oracle(B, H, W, mode, d):
    ws = 14 if not (H == 16 and mode == "window") else 8
    cfg = L.make_cfg(B, H, W, mode, ws, 2, 64, d)
    p = L.sparsesam_pattern(cfg)
    geo = O.Geometry(B, H, W, mode, ws)
    op = O.pattern(geo.unit_tokens, d)
    assert (p.units, p.unit_tokens) == (geo.units, geo.unit_tokens)
    assert (p.L, p.b, p.nb, p.W, p.g) == (op.L, op.b, op.nb, op.W, op.g)
    assert p.rho == op.rho
    assert p.keep == O.keep_count(d, H * W)
    row_ptr, col_idx = L.sparsesam_blocklist(cfg)
    assert row_ptr == list(op.row_ptr) and col_idx == list(op.col_idx)


@pytest.mark.parametrize("d", [x / 100 for x in range(1, 101, 3)] + [0.4, 0.3, 0.5, 1.0])
def test_keep_count_and_band_choice_sweep(d):
    for h, w in ((4, 4), (14, 14), (16, 16), (32, 32), (64, 64)):
        T = h * w
        cfg = L.make_cfg(1, h, w, "global", 14, 1, 64, d)
        p = L.sparsesam_pattern(cfg)
        assert p.keep == O.keep_count(d, T)
        assert p.W == O.pattern(T, d).W


# ---- host-side validation (no GPU is touched: every case fails before any CUDA call) ----------
FAKE = 1 << 20      # an aligned, never-dereferenced address


def test_validation_codes():
    good = L.make_cfg(1, 16, 16, "global", 14, 1, 64, 0.4)
    lib = L.lib
    by = ctypes.byref
    # bad density / shapes
    for d in (0.0, -0.5, 1.5, float("nan")):
        assert lib.sparsesam_pattern(by(L.make_cfg(1, 16, 16, density=d)), by(L.SsPattern())) == L.SS_EINVAL
    assert lib.sparsesam_pattern(by(L.make_cfg(0, 16, 16, density=0.4)), by(L.SsPattern())) == L.SS_EINVAL
    assert lib.sparsesam_pattern(by(L.make_cfg(1, 5, 5, density=0.4)), by(L.SsPattern())) == L.SS_EUNSUPPORTED
    assert lib.sparsesam_pattern(by(L.make_cfg(1, 2, 2, density=0.4)), by(L.SsPattern())) == L.SS_EUNSUPPORTED
    assert lib.sparsesam_pattern(None, by(L.SsPattern())) == L.SS_EINVAL
    assert lib.sparsesam_pattern(by(L.make_cfg(1, 16, 16, "window", 0, density=0.4)), by(L.SsPattern())) == L.SS_EINVAL
    # null pointers
    assert lib.sparsesam_score(by(good), None, FAKE, None) == L.SS_EINVAL
    assert lib.sparsesam_perm(by(good), FAKE, None, None, None, None) == L.SS_EINVAL
    assert lib.sparsesam_score_perm(by(good), None, FAKE, FAKE, None, None, None) == L.SS_EINVAL
    assert lib.sparsesam_score_perm(by(good), FAKE, None, FAKE, None, None, None) == L.SS_EINVAL
    assert lib.sparsesam_score_perm(by(good), FAKE, FAKE, None, None, None, None) == L.SS_EINVAL
    assert lib.sparsesam_block_workspace(None, 64, 256) == 0
    assert lib.sparsesam_block_workspace(by(good), 0, 256) == 0
    assert lib.sparsesam_block_workspace(by(good), 64, 256) >= (
        lib.sparsesam_attn_workspace(by(good))
        + lib.sparsesam_rcmlp_workspace(by(good), 64, 256, O.keep_count(0.4, 256)))
    blk = [FAKE] * 5 + [64, 256] + [FAKE] * 4 + [FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, None]
    assert lib.sparsesam_block(by(good), *blk) == L.SS_EWORKSPACE   # 1 byte of workspace
    for i in (0, 1, 11, 12, 14, 15):   # lum, q, score, perm, keep, out
        bad = list(blk)
        bad[i] = None
        assert lib.sparsesam_block(by(good), *bad) == L.SS_EINVAL, i
    overlap = list(blk)
    overlap[17] = 1 << 30   # enough workspace: the x / out overlap is what is refused
    assert overlap[4] == overlap[15]   # x and out are the same fake buffer
    assert lib.sparsesam_block(by(good), *overlap) == L.SS_EINVAL
    assert lib.sparsesam_attn(by(good), None, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == L.SS_EINVAL
    # unsupported head_dim
    bad_dh = L.make_cfg(1, 16, 16, "global", 14, 1, 96, 0.4)
    assert lib.sparsesam_attn(by(bad_dh), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == L.SS_EUNSUPPORTED
    # misaligned q
    assert lib.sparsesam_attn(by(good), FAKE + 2, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == L.SS_EINVAL
    # workspace too small / misaligned / missing
    need = L.sparsesam_attn_workspace(good)
    assert need == 3 * 256 * 64 * 2
    assert lib.sparsesam_attn(by(good), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, None) == L.SS_EWORKSPACE
    assert lib.sparsesam_attn(by(good), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 16, need, None) == L.SS_EWORKSPACE
    assert lib.sparsesam_attn(by(good), FAKE, FAKE, FAKE, FAKE, FAKE, None, need, None) == L.SS_EWORKSPACE
    # rcmlp: C not a multiple of 64, K outside [0, T], workspace
    K = O.keep_count(0.4, 256)
    assert lib.sparsesam_rcmlp(by(good), FAKE, 48, 256, FAKE, None, FAKE, None, FAKE, K, FAKE, 1 << 30, None) == L.SS_EUNSUPPORTED
    for badK in (-1, 257):
        assert lib.sparsesam_rcmlp(by(good), FAKE, 64, 256, FAKE, None, FAKE, None, FAKE, badK, FAKE, 1 << 30, None) == L.SS_EINVAL
        assert lib.sparsesam_rcmlp_workspace(by(good), 64, 256, badK) == 0
    need_m = L.sparsesam_rcmlp_workspace(good, 64, 256, K)
    assert need_m == math.ceil(K * 64 * 2 / 256) * 256 + math.ceil(K * 256 * 2 / 256) * 256
    assert lib.sparsesam_rcmlp(by(good), FAKE, 64, 256, FAKE, None, FAKE, None, FAKE, K, FAKE, need_m - 1, None) == L.SS_EWORKSPACE
    # a caller K other than the density's (another keep criterion) sizes the workspace by that K
    assert L.sparsesam_rcmlp_workspace(good, 64, 256, 200) > need_m
    # K = 0: every row is residual; nothing is launched, even without a workspace
    assert lib.sparsesam_rcmlp(by(good), FAKE, 64, 256, FAKE, None, FAKE, None, FAKE, 0, None, 0, None) == L.SS_OK
    # A long-K fc2 (ViT-H: K = 5120, 80 k-blocks; 4 images, 4916 kept rows) has a last partial
    # round of tiles split in two along K: the workspace holds their fp32 halves and counters
    # beyond xk and H.
    vith = L.make_cfg(4, 64, 64, "global", 14, 16, 80, 0.3)
    M = 4 * O.keep_count(0.3, 4096)
    xk_h = math.ceil(M * 1280 * 2 / 256) * 256 + math.ceil(M * 5120 * 2 / 256) * 256
    # 47 tail tiles of 128 x 256 fp32 (6.2 MB), where a two-way split of all 195 tiles would need
    # 51 MB of partials
    extra = L.sparsesam_rcmlp_workspace(vith, 1280, 5120, O.keep_count(0.3, 4096)) - xk_h
    assert 47 * 128 * 256 * 4 <= extra < 8 << 20
    # variants: missing outputs, K outside [0, T], C not a multiple of 8, misaligned delta
    assert lib.sparsesam_random_perm(by(good), 1, None, FAKE, None, None, None) == L.SS_EINVAL
    assert lib.sparsesam_random_perm(by(good), 1, FAKE, None, None, None, None) == L.SS_EINVAL
    assert lib.sparsesam_keep_by_update(by(good), FAKE, 64, 257, FAKE, FAKE, None) == L.SS_EINVAL
    assert lib.sparsesam_keep_by_update(by(good), FAKE, 64, -1, FAKE, FAKE, None) == L.SS_EINVAL
    assert lib.sparsesam_keep_by_update(by(good), FAKE, 60, 10, FAKE, FAKE, None) == L.SS_EUNSUPPORTED
    assert lib.sparsesam_keep_by_update(by(good), FAKE + 2, 64, 10, FAKE, FAKE, None) == L.SS_EINVAL
    assert lib.sparsesam_keep_by_update(by(good), None, 64, 10, FAKE, FAKE, None) == L.SS_EINVAL
    assert lib.sparsesam_keep_by_update(by(good), FAKE, 64, 0, FAKE, FAKE, None) == L.SS_OK
    # blocklist capacity
    rp = (ctypes.c_int32 * 8)()
    ci = (ctypes.c_int32 * 2)()
    assert lib.sparsesam_blocklist(by(good), ctypes.cast(rp, ctypes.c_void_p), ctypes.cast(ci, ctypes.c_void_p), 2) == L.SS_EINVAL
    # trace records outside the range
    name, ms = ctypes.c_char_p(), ctypes.c_float()
    assert lib.sparsesam_trace_get(0, by(name), by(ms)) == L.SS_EINVAL
    assert L.sparsesam_launch_count() == 0


def test_encoder_block_and_stack_validation():
    lib = L.lib
    by = ctypes.byref
    cfg = L.make_cfg(1, 16, 16, "global", 14, 2, 64, 0.4)        # C = 128
    K = O.keep_count(0.4, 256)
    need = L.sparsesam_encoder_block_workspace(cfg, 128, 512, K)
    # LN1 rows + the attention's workspace + the RC-MLP's workspace at least
    assert need >= 256 * 128 * 2 + L.sparsesam_attn_workspace(cfg) + L.sparsesam_rcmlp_workspace(cfg, 128, 512, K)
    assert L.sparsesam_encoder_block_workspace(cfg, 128, 512, 0) < need
    assert L.sparsesam_encoder_block_workspace(cfg, 128, 512, 257) == 0
    w = L.SsBlockWeights(**{n: FAKE for n in L.BLOCK_WEIGHT_FIELDS})

    def call(c=cfg, x=FAKE, C=128, hidden=512, wt=w, perm=FAKE, inv=FAKE, keep=FAKE, k=K, ws=FAKE,
             nbytes=1):
        return lib.sparsesam_encoder_block(by(c), x, C, hidden, by(wt), perm, inv, keep, k, ws,
                                           nbytes, None)
    assert call() == L.SS_EWORKSPACE                               # 1 byte of workspace
    assert call(ws=FAKE + 16, nbytes=1 << 30) == L.SS_EWORKSPACE   # misaligned workspace
    assert call(C=192) == L.SS_EINVAL                              # C != heads * head_dim
    assert call(hidden=500) == L.SS_EUNSUPPORTED
    assert call(c=L.make_cfg(1, 16, 16, "global", 14, 2, 96, 0.4), C=192) == L.SS_EUNSUPPORTED
    assert call(c=L.make_cfg(1, 16, 16, "global", 14, 3, 80, 0.4), C=240) == L.SS_EUNSUPPORTED
    assert call(x=None) == L.SS_EINVAL
    assert call(x=FAKE + 2) == L.SS_EINVAL
    assert call(perm=None) == L.SS_EINVAL
    assert call(inv=None) == L.SS_EINVAL
    assert call(keep=None) == L.SS_EINVAL
    assert call(k=-1) == L.SS_EINVAL and call(k=257) == L.SS_EINVAL
    for n in ("ln1_w", "ln1_b", "w_qkv", "w_proj", "ln2_w", "ln2_b", "w1", "w2"):
        bad = L.SsBlockWeights(**{f: (None if f == n else FAKE) for f in L.BLOCK_WEIGHT_FIELDS})
        assert call(wt=bad) == L.SS_EINVAL, n
    for n in ("b_qkv", "b_proj", "b1", "b2"):                      # Linear biases are optional
        nob = L.SsBlockWeights(**{f: (None if f == n else FAKE) for f in L.BLOCK_WEIGHT_FIELDS})
        assert call(wt=nob) == L.SS_EWORKSPACE, n
        mis = L.SsBlockWeights(**{f: (FAKE + 8 if f == n else FAKE) for f in L.BLOCK_WEIGHT_FIELDS})
        assert call(wt=mis) == L.SS_EINVAL, n
    # the stack: its workspace holds both geometries' rankings and the larger block workspace
    sw = L.sparsesam_encoder_stack_workspace(cfg, 128, 512)
    cw = L.make_cfg(1, 16, 16, "window", 14, 2, 64, 0.4)           # 2 x 2 windows of 196
    assert sw > max(need, L.sparsesam_encoder_block_workspace(cw, 128, 512, K))
    arr = (L.SsBlockWeights * 2)(w, w)
    flags = (ctypes.c_uint8 * 2)(0, 1)

    def stack(lum=FAKE, n=2, ws=FAKE, nbytes=1 << 40, warr=arr):
        return lib.sparsesam_encoder_stack(by(cfg), lum, FAKE, 128, 512, n, warr,
                                           ctypes.addressof(flags), ws, nbytes, None)
    assert stack(nbytes=sw - 1) == L.SS_EWORKSPACE
    assert stack(lum=None) == L.SS_EINVAL
    assert stack(n=-1) == L.SS_EINVAL
    bad = L.SsBlockWeights(**{f: (None if f == "w_proj" else FAKE) for f in L.BLOCK_WEIGHT_FIELDS})
    assert stack(warr=(L.SsBlockWeights * 2)(w, bad)) == L.SS_EINVAL   # checked before any launch
    assert L.sparsesam_launch_count() == 0


def test_relpos_and_partial_validation():
    lib = L.lib
    by = ctypes.byref
    g = L.make_cfg(1, 16, 16, "global", 14, 2, 64, 0.4)
    need = L.sparsesam_attn_relpos_workspace(g)
    # the pair kernel's workspace, the stacked tables, the bias products (fp16, 2*(31+31)->64
    # columns per row), the key offsets
    assert need >= L.sparsesam_attn_workspace(g) + 2 * 256 * 64 * 2

    def rel(cfg=g, rh=FAKE, rw=FAKE, nbytes=1 << 40):
        return lib.sparsesam_attn_relpos(by(cfg), FAKE, FAKE, FAKE, FAKE, rh, rw, FAKE, FAKE,
                                         nbytes, None)
    assert rel(nbytes=need - 1) == L.SS_EWORKSPACE
    assert rel(rh=None) == L.SS_EINVAL and rel(rw=FAKE + 2) == L.SS_EINVAL
    assert rel(cfg=L.make_cfg(1, 16, 16, "global", 14, 2, 80, 0.4)) == L.SS_EUNSUPPORTED
    assert rel(cfg=L.make_cfg(1, 80, 64, "global", 14, 2, 64, 0.4)) == L.SS_EUNSUPPORTED   # 80 + 64 > 128

    def part(cfg=g, prefix=1, base=10000.0, nbytes=1 << 40):
        return lib.sparsesam_attn_partial(by(cfg), prefix, base, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                          nbytes, None)
    pneed = L.sparsesam_attn_partial_workspace(g, 1)
    assert pneed > L.sparsesam_attn_workspace(g)
    assert part(nbytes=pneed - 1) == L.SS_EWORKSPACE
    assert part(prefix=-1) == L.SS_EINVAL and part(prefix=5) == L.SS_EINVAL
    assert part(base=0.5) == L.SS_EINVAL and part(base=float("inf")) == L.SS_EINVAL
    assert part(cfg=L.make_cfg(1, 16, 16, "window", 14, 2, 64, 0.4)) == L.SS_EUNSUPPORTED
    assert part(cfg=L.make_cfg(1, 16, 16, "global", 14, 33, 64, 0.4)) == L.SS_EUNSUPPORTED
    assert L.sparsesam_launch_count() == 0


def test_binding_raises_on_error():
    with pytest.raises(L.SparseSAMError) as e:
        L.sparsesam_pattern(L.make_cfg(1, 5, 5, density=0.4))
    assert e.value.code == L.SS_EUNSUPPORTED
