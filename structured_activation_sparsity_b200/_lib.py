"""ctypes binding of libsparsesam.so (the C ABI in include/sparsesam.h).

Argument marshalling only: every step of the hot path runs in the library's sm_100a kernels. Tensor
arguments may be torch tensors (their data_ptr() is passed) or raw integer addresses. There is no
fallback: if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparsesam.so")

SS_OK = 0
SS_EINVAL = -1
SS_EUNSUPPORTED = -2
SS_EWORKSPACE = -3
SS_ECUDA = -4
SS_ETIMEOUT = -5
SS_EINDEX = -6
SS_GLOBAL = 0
SS_WINDOW = 1


class SsCfg(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("window", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("density", ctypes.c_double)]


class SsPattern(ctypes.Structure):
    _fields_ = [("units", ctypes.c_int32), ("unit_tokens", ctypes.c_int32),
                ("stripes", ctypes.c_int32), ("L", ctypes.c_int32), ("b", ctypes.c_int32),
                ("nb", ctypes.c_int32), ("W", ctypes.c_int32), ("g", ctypes.c_int32),
                ("nnz", ctypes.c_int32), ("keep", ctypes.c_int32), ("rho", ctypes.c_double)]


BLOCK_WEIGHT_FIELDS = ("ln1_w", "ln1_b", "w_qkv", "b_qkv", "w_proj", "b_proj", "ln2_w", "ln2_b",
                       "w1", "b1", "w2", "b2")


class SsBlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in BLOCK_WEIGHT_FIELDS]


class SparseSAMError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({strerror(code)})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m structured_activation_sparsity_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, VP = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p
    cfgp = ctypes.POINTER(SsCfg)
    sig = {
        "sparsesam_pattern": (ctypes.c_int, [cfgp, ctypes.POINTER(SsPattern)]),
        "sparsesam_blocklist": (ctypes.c_int, [cfgp, P, P, I32]),
        "sparsesam_score": (ctypes.c_int, [cfgp, P, P, VP]),
        "sparsesam_perm": (ctypes.c_int, [cfgp, P, P, P, P, VP]),
        "sparsesam_score_perm": (ctypes.c_int, [cfgp, P, P, P, P, P, VP]),
        "sparsesam_random_perm": (ctypes.c_int, [cfgp, ctypes.c_uint64, P, P, P, P, VP]),
        "sparsesam_keep_by_update": (ctypes.c_int, [cfgp, P, I32, I32, P, P, VP]),
        "sparsesam_block_workspace": (SZ, [cfgp, I32, I32]),
        "sparsesam_block": (ctypes.c_int, [cfgp, P, P, P, P, P, I32, I32, P, P, P, P, P, P, P, P,
                                           P, P, SZ, VP]),
        "sparsesam_attn_workspace": (SZ, [cfgp]),
        "sparsesam_attn": (ctypes.c_int, [cfgp, P, P, P, P, P, P, SZ, VP]),
        "sparsesam_attn_gathered": (ctypes.c_int, [cfgp, P, SZ, P, P, VP]),
        "sparsesam_rcmlp_workspace": (SZ, [cfgp, I32, I32, I32]),
        "sparsesam_rcmlp": (ctypes.c_int, [cfgp, P, I32, I32, P, P, P, P, P, I32, P, SZ, VP]),
        "sparsesam_rcmlp_noalloc": (ctypes.c_int, [cfgp, P, I32, I32, P, P, P, P, P, I32, VP]),
        "sparsesam_attn_relpos_workspace": (SZ, [cfgp]),
        "sparsesam_attn_relpos": (ctypes.c_int, [cfgp, P, P, P, P, P, P, P, P, SZ, VP]),
        "sparsesam_attn_partial_workspace": (SZ, [cfgp, I32]),
        "sparsesam_attn_partial": (ctypes.c_int, [cfgp, I32, ctypes.c_float, P, P, P, P, P, P, SZ,
                                                  VP]),
        "sparsesam_encoder_block_workspace": (SZ, [cfgp, I32, I32, I32]),
        "sparsesam_encoder_block": (ctypes.c_int, [cfgp, P, I32, I32, ctypes.POINTER(SsBlockWeights),
                                                   P, P, P, I32, P, SZ, VP]),
        "sparsesam_encoder_stack_workspace": (SZ, [cfgp, I32, I32]),
        "sparsesam_encoder_stack": (ctypes.c_int, [cfgp, P, P, I32, I32, I32,
                                                   ctypes.POINTER(SsBlockWeights), P, P, SZ, VP]),
        "sparsesam_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
        "sparsesam_wait_selftest": (ctypes.c_int, [I32, VP]),
        "sparsesam_device_status": (ctypes.c_int, [ctypes.POINTER(I32), VP]),
        "sparsesam_launch_count": (ctypes.c_uint64, []),
        "sparsesam_trace_start": (ctypes.c_int, [I32]),
        "sparsesam_trace_stop": (ctypes.c_int, []),
        "sparsesam_trace_get": (ctypes.c_int, [I32, ctypes.POINTER(ctypes.c_char_p),
                                               ctypes.POINTER(ctypes.c_float)]),
        "sparsesam_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def strerror(code: int) -> str:
    return lib.sparsesam_strerror(int(code)).decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream  # torch.cuda.Stream


def _check(fn: str, rc: int) -> int:
    if rc != SS_OK:
        raise SparseSAMError(fn, rc)
    return rc


def make_cfg(batch, grid_h, grid_w, mode="global", window=14, heads=1, head_dim=64,
             density=1.0) -> SsCfg:
    m = SS_GLOBAL if mode in ("global", SS_GLOBAL) else SS_WINDOW
    return SsCfg(batch, grid_h, grid_w, m, window, heads, head_dim, float(density))


def cfg_for(wl, density: float | None = None) -> SsCfg:
    """SsCfg of a workloads.Workload."""
    return make_cfg(wl.batch, wl.grid_h, wl.grid_w, wl.mode, wl.window, wl.heads, wl.head_dim,
                    wl.density if density is None else density)


def sparsesam_pattern(cfg: SsCfg) -> SsPattern:
    p = SsPattern()
    _check("sparsesam_pattern", lib.sparsesam_pattern(ctypes.byref(cfg), ctypes.byref(p)))
    return p


def sparsesam_blocklist(cfg: SsCfg):
    """(row_ptr, col_idx) as Python int lists."""
    p = sparsesam_pattern(cfg)
    row_ptr = (ctypes.c_int32 * (p.nb + 1))()
    col_idx = (ctypes.c_int32 * max(1, p.nnz))()
    _check("sparsesam_blocklist",
           lib.sparsesam_blocklist(ctypes.byref(cfg), ctypes.cast(row_ptr, ctypes.c_void_p),
                                   ctypes.cast(col_idx, ctypes.c_void_p), p.nnz))
    return list(row_ptr), list(col_idx)[:p.nnz]


def sparsesam_score(cfg, lum, score, stream=None):
    return _check("sparsesam_score",
                  lib.sparsesam_score(ctypes.byref(cfg), _ptr(lum), _ptr(score), _stream(stream)))


def sparsesam_perm(cfg, score, perm, inv, keep, stream=None):
    return _check("sparsesam_perm",
                  lib.sparsesam_perm(ctypes.byref(cfg), _ptr(score), _ptr(perm), _ptr(inv),
                                     _ptr(keep), _stream(stream)))


def sparsesam_score_perm(cfg, lum, score, perm, inv, keep, stream=None):
    return _check("sparsesam_score_perm",
                  lib.sparsesam_score_perm(ctypes.byref(cfg), _ptr(lum), _ptr(score), _ptr(perm),
                                           _ptr(inv), _ptr(keep), _stream(stream)))


def sparsesam_random_perm(cfg, seed, score, perm, inv, keep, stream=None):
    """S2 over seeded random scores (the random-permutation ablation)."""
    return _check("sparsesam_random_perm",
                  lib.sparsesam_random_perm(ctypes.byref(cfg), int(seed), _ptr(score), _ptr(perm),
                                            _ptr(inv), _ptr(keep), _stream(stream)))


def sparsesam_keep_by_update(cfg, delta, C, K, mag, keep, stream=None):
    """The keep list of the K tokens with the largest update magnitude sum_c delta[b,t,c]^2."""
    return _check("sparsesam_keep_by_update",
                  lib.sparsesam_keep_by_update(ctypes.byref(cfg), _ptr(delta), int(C), int(K),
                                               _ptr(mag), _ptr(keep), _stream(stream)))


def sparsesam_block_workspace(cfg, C, hidden) -> int:
    return int(lib.sparsesam_block_workspace(ctypes.byref(cfg), C, hidden))


def sparsesam_block(cfg, lum, q, k, v, x, C, hidden, w1, b1, w2, b2, score, perm, inv, keep, out,
                    ws, ws_bytes, stream=None):
    return _check("sparsesam_block",
                  lib.sparsesam_block(ctypes.byref(cfg), _ptr(lum), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(x), C, hidden, _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2),
                                      _ptr(score), _ptr(perm), _ptr(inv), _ptr(keep), _ptr(out),
                                      _ptr(ws), ws_bytes, _stream(stream)))


def sparsesam_attn_workspace(cfg) -> int:
    return int(lib.sparsesam_attn_workspace(ctypes.byref(cfg)))


def sparsesam_attn(cfg, q, k, v, perm, out, ws, ws_bytes, stream=None):
    return _check("sparsesam_attn",
                  lib.sparsesam_attn(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(perm),
                                     _ptr(out), _ptr(ws), int(ws_bytes), _stream(stream)))


def sparsesam_attn_gathered(cfg, ws, ws_bytes, perm, out, stream=None):
    """The attention kernel alone over the permuted Q, K, V an earlier sparsesam_attn left in ws."""
    return _check("sparsesam_attn_gathered",
                  lib.sparsesam_attn_gathered(ctypes.byref(cfg), _ptr(ws), int(ws_bytes), _ptr(perm),
                                              _ptr(out), _stream(stream)))


def sparsesam_rcmlp_workspace(cfg, C: int, hidden: int, K: int) -> int:
    return int(lib.sparsesam_rcmlp_workspace(ctypes.byref(cfg), int(C), int(hidden), int(K)))


def sparsesam_rcmlp(cfg, x, C, hidden, w1, b1, w2, b2, keep, K, ws, ws_bytes, stream=None):
    return _check("sparsesam_rcmlp",
                  lib.sparsesam_rcmlp(ctypes.byref(cfg), _ptr(x), int(C), int(hidden), _ptr(w1),
                                      _ptr(b1), _ptr(w2), _ptr(b2), _ptr(keep), int(K), _ptr(ws),
                                      int(ws_bytes), _stream(stream)))


def sparsesam_rcmlp_noalloc(cfg, x, C, hidden, w1, b1, w2, b2, keep, K, stream=None):
    """sparsesam_rcmlp with its scratch in the library's fixed 32 MiB device array (no workspace
    argument, nothing allocated). For callers that cannot allocate device memory."""
    return _check("sparsesam_rcmlp_noalloc",
                  lib.sparsesam_rcmlp_noalloc(ctypes.byref(cfg), _ptr(x), int(C), int(hidden),
                                              _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(keep),
                                              int(K), _stream(stream)))


def sparsesam_attn_relpos_workspace(cfg) -> int:
    return int(lib.sparsesam_attn_relpos_workspace(ctypes.byref(cfg)))


def sparsesam_attn_relpos(cfg, q, k, v, perm, rel_h, rel_w, out, ws, ws_bytes, stream=None):
    """S3 with SAM's decomposed relative-position bias (rel_h [2Hu-1, dh], rel_w [2Wu-1, dh])."""
    return _check("sparsesam_attn_relpos",
                  lib.sparsesam_attn_relpos(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(perm), _ptr(rel_h), _ptr(rel_w), _ptr(out),
                                            _ptr(ws), int(ws_bytes), _stream(stream)))


def sparsesam_attn_partial_workspace(cfg, prefix) -> int:
    return int(lib.sparsesam_attn_partial_workspace(ctypes.byref(cfg), int(prefix)))


def sparsesam_attn_partial(cfg, prefix, rope_base, q, k, v, perm, out, ws, ws_bytes, stream=None):
    """S3 over prefix + patch tokens with 2-D RoPE on the patch tokens (rope_base 0: none)."""
    return _check("sparsesam_attn_partial",
                  lib.sparsesam_attn_partial(ctypes.byref(cfg), int(prefix), float(rope_base),
                                             _ptr(q), _ptr(k), _ptr(v), _ptr(perm), _ptr(out),
                                             _ptr(ws), int(ws_bytes), _stream(stream)))


def block_weights(w) -> SsBlockWeights:
    """An ss_block_weights of device pointers from a mapping name -> tensor (or None / address)."""
    return SsBlockWeights(**{n: _ptr(w.get(n)) for n in BLOCK_WEIGHT_FIELDS})


def sparsesam_encoder_block_workspace(cfg, C, hidden, K) -> int:
    return int(lib.sparsesam_encoder_block_workspace(ctypes.byref(cfg), int(C), int(hidden), int(K)))


def sparsesam_encoder_block(cfg, x, C, hidden, weights, perm, inv, keep, K, ws, ws_bytes,
                            stream=None):
    """One full encoder block in place on x; weights: an SsBlockWeights or a mapping name ->
    tensor."""
    w = weights if isinstance(weights, SsBlockWeights) else block_weights(weights)
    return _check("sparsesam_encoder_block",
                  lib.sparsesam_encoder_block(ctypes.byref(cfg), _ptr(x), int(C), int(hidden),
                                              ctypes.byref(w), _ptr(perm), _ptr(inv), _ptr(keep),
                                              int(K), _ptr(ws), int(ws_bytes), _stream(stream)))


def sparsesam_encoder_stack_workspace(cfg, C, hidden) -> int:
    return int(lib.sparsesam_encoder_stack_workspace(ctypes.byref(cfg), int(C), int(hidden)))


def sparsesam_encoder_stack(cfg, lum, x, C, hidden, weights, is_global, ws, ws_bytes,
                            stream=None):
    """The encoder's blocks in order over x; weights: a list of SsBlockWeights or mappings,
    is_global: one flag per block."""
    n = len(weights)
    if len(is_global) != n:
        raise ValueError("one is_global flag per block")
    arr = (SsBlockWeights * max(n, 1))(*[w if isinstance(w, SsBlockWeights) else block_weights(w)
                                          for w in weights])
    flags = (ctypes.c_uint8 * max(n, 1))(*[1 if g else 0 for g in is_global])
    return _check("sparsesam_encoder_stack",
                  lib.sparsesam_encoder_stack(ctypes.byref(cfg), _ptr(lum), _ptr(x), int(C),
                                              int(hidden), n, arr, ctypes.addressof(flags),
                                              _ptr(ws), int(ws_bytes), _stream(stream)))


def sparsesam_set_wait_limit_ns(ns: int):
    """Test support: the device waits' time limit on the current device (0 = the default)."""
    return _check("sparsesam_set_wait_limit_ns", lib.sparsesam_set_wait_limit_ns(int(ns)))


def sparsesam_wait_selftest(which: int, stream=None):
    """Test support: one bounded device wait that runs out (which 0: mbarrier, 1: counter) or is
    satisfied (2, 3)."""
    return _check("sparsesam_wait_selftest",
                  lib.sparsesam_wait_selftest(int(which), _stream(stream)))


def sparsesam_device_status(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check("sparsesam_device_status", lib.sparsesam_device_status(ctypes.byref(v), _stream(stream)))
    return v.value


def sparsesam_launch_count() -> int:
    return int(lib.sparsesam_launch_count())


def sparsesam_trace_start(capacity: int):
    return _check("sparsesam_trace_start", lib.sparsesam_trace_start(int(capacity)))


def sparsesam_trace_stop():
    """Returns [(kernel name, ms), ...] for the launches recorded since trace_start."""
    n = lib.sparsesam_trace_stop()
    if n < 0:
        raise SparseSAMError("sparsesam_trace_stop", n)
    out = []
    for i in range(n):
        name, ms = ctypes.c_char_p(), ctypes.c_float()
        _check("sparsesam_trace_get", lib.sparsesam_trace_get(i, ctypes.byref(name), ctypes.byref(ms)))
        out.append((name.value.decode(), float(ms.value)))
    return out
