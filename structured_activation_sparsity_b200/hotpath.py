"""One encoder block's hot path over device buffers: score -> perm -> attn -> rcmlp.

PyTorch only allocates the device memory and supplies the stream; each step is one call into the
C ABI (libsparsesam.so).
"""
from __future__ import annotations

import torch

from . import _lib as L


class HotPath:
    """Device buffers for one workload and the four library calls over them."""

    def __init__(self, wl, device="cuda", density: float | None = None, bias: bool = True):
        self.wl = wl
        self.cfg = L.cfg_for(wl, density)
        self.pattern = L.sparsesam_pattern(self.cfg)
        self.K = self.pattern.keep
        dev = torch.device(device)
        B, T, C, Hd = wl.batch, wl.tokens_per_image, wl.dim, wl.hidden
        U, N, H, D = wl.units, wl.unit_tokens, wl.heads, wl.head_dim
        e = dict(device=dev)
        self.lum = torch.empty((B, wl.grid_h, wl.grid_w), dtype=torch.float32, **e)
        self.score = torch.empty((B, T), dtype=torch.float64, **e)
        self.perm = torch.empty((U, N), dtype=torch.int32, **e)
        self.inv = torch.empty((U, N), dtype=torch.int32, **e)
        self.keep = torch.empty((B, self.K), dtype=torch.int32, **e)
        self.q = torch.empty((U, N, H, D), dtype=torch.bfloat16, **e)
        self.k = torch.empty_like(self.q)
        self.v = torch.empty_like(self.q)
        self.out = torch.empty_like(self.q)
        self.x = torch.empty((B, T, C), dtype=torch.bfloat16, **e)
        self.w1 = torch.empty((Hd, C), dtype=torch.bfloat16, **e)
        self.w2 = torch.empty((C, Hd), dtype=torch.bfloat16, **e)
        self.b1 = torch.zeros((Hd,), dtype=torch.bfloat16, **e) if bias else None
        self.b2 = torch.zeros((C,), dtype=torch.bfloat16, **e) if bias else None
        # One workspace for the whole-block call; the per-step calls use its two parts (the
        # attention's first, 256-byte aligned, then the MLP's).
        self.ws_attn_bytes = L.sparsesam_attn_workspace(self.cfg)
        self.ws_mlp_bytes = L.sparsesam_rcmlp_workspace(self.cfg, C, Hd, self.K)
        self.ws_block_bytes = L.sparsesam_block_workspace(self.cfg, C, Hd)
        self.ws_block = torch.empty((self.ws_block_bytes,), dtype=torch.uint8, **e)
        attn_part = -(-self.ws_attn_bytes // 256) * 256
        self.ws_attn = self.ws_block[:attn_part]
        self.ws_mlp = self.ws_block[attn_part:]

    # -- inputs --------------------------------------------------------------------------------
    def load(self, lum, q, k, v, x, w1, b1, w2, b2):
        """Copy inputs (CPU or device tensors; bf16 where the buffer is bf16) into the buffers."""
        for dst, src in ((self.lum, lum), (self.q, q), (self.k, k), (self.v, v), (self.x, x),
                         (self.w1, w1), (self.w2, w2), (self.b1, b1), (self.b2, b2)):
            if dst is not None and src is not None:
                dst.copy_(src)

    def input_tensors(self):
        return [self.lum, self.q, self.k, self.v, self.x]

    # -- the four steps ------------------------------------------------------------------------
    def score_step(self, stream=None):
        L.sparsesam_score(self.cfg, self.lum, self.score, stream)

    def perm_step(self, stream=None):
        L.sparsesam_perm(self.cfg, self.score, self.perm, self.inv, self.keep, stream)

    def score_perm_step(self, stream=None):
        """S1 and S2 in one pass (the same score, perm, inv and keep as score_step + perm_step)."""
        L.sparsesam_score_perm(self.cfg, self.lum, self.score, self.perm, self.inv, self.keep,
                               stream)

    def attn_step(self, stream=None):
        L.sparsesam_attn(self.cfg, self.q, self.k, self.v, self.perm, self.out, self.ws_attn,
                         self.ws_attn_bytes, stream)

    def attn_kernel_step(self, stream=None):
        """The attention kernel alone over the permuted Q, K, V the last attn_step / step left in
        the workspace (for timing the kernel by itself)."""
        L.sparsesam_attn_gathered(self.cfg, self.ws_attn, self.ws_attn_bytes, self.perm, self.out,
                                  stream)

    def mlp_step(self, stream=None):
        L.sparsesam_rcmlp(self.cfg, self.x, self.wl.dim, self.wl.hidden, self.w1, self.b1,
                          self.w2, self.b2, self.keep, self.K, self.ws_mlp, self.ws_mlp_bytes,
                          stream)

    def step(self, stream=None):
        """S1..S4 of one block, asynchronously on `stream` (a torch.cuda.Stream or None), in the
        whole-block call (S1 and S2 as one fused pass)."""
        L.sparsesam_block(self.cfg, self.lum, self.q, self.k, self.v, self.x, self.wl.dim,
                          self.wl.hidden, self.w1, self.b1, self.w2, self.b2, self.score, self.perm,
                          self.inv, self.keep, self.out, self.ws_block, self.ws_block_bytes, stream)

    def step_by_calls(self, stream=None):
        """The same step through the per-step calls (S1+S2 fused, then S3, then S4)."""
        self.score_perm_step(stream)
        self.attn_step(stream)
        self.mlp_step(stream)
