"""Seeded synthetic inputs for the SparseSAM hot path.

These stand in for SA-1B / HQ-44K / COCO images and SAM checkpoints, which the pages evaluate on and
which are not available here. The same arrays feed the float64 oracle and the CUDA path. This module
draws random numbers and rounds them to bf16; it holds none of the method's arithmetic.

Recipe:
  * luminance: one background level ~ U(0,1) per image; 12 discs painted in order, each with radius
    ~ U(2, Hg/4), centre ~ U(grid), level ~ U(0,1); then i.i.d. N(0, 0.05) noise. Piecewise-constant
    regions with edges, like a natural image's luminance at token resolution.
  * q, k, v ~ N(0,1) · qkv_scale, layout [U, N, heads, dh].
  * x ~ N(0,1) [B, Hg·Wg, C]; W1 [hidden, C] and W2 [C, hidden] ~ N(0, 0.02); biases 0 unless asked.
  * full encoder blocks (block_params): every Linear weight [out, in] ~ N(0, 1/in) (so that each
    branch of the block adds O(1) values to the residual stream), its bias ~ N(0, 0.1^2); LayerNorm
    weights ~ 1 + N(0, 0.1^2), LayerNorm biases ~ N(0, 0.1^2).
Every tensor has its own stream: numpy PCG64 seeded with (workload seed, tensor tag[, block]).
"""
from __future__ import annotations

import numpy as np
import torch

from .workloads import Workload

_TAGS = {"lum": 1, "q": 2, "k": 3, "v": 4, "x": 5, "w1": 6, "b1": 7, "w2": 8, "b2": 9,
         "ln1_w": 10, "ln1_b": 11, "w_qkv": 12, "b_qkv": 13, "w_proj": 14, "b_proj": 15,
         "ln2_w": 16, "ln2_b": 17}


def rng(seed: int, tag: str, block: int | None = None) -> np.random.Generator:
    key = [int(seed), _TAGS[tag]] + ([] if block is None else [int(block)])
    return np.random.default_rng(key)


def luminance(wl: Workload, seed: int | None = None, discs: int = 12, noise: float = 0.05) -> np.ndarray:
    """fp32 [B, Hg, Wg] blob-plus-noise luminance map."""
    g = rng(wl.seed if seed is None else seed, "lum")
    H, W = wl.grid_h, wl.grid_w
    yy, xx = np.meshgrid(np.arange(H, dtype=np.float64), np.arange(W, dtype=np.float64), indexing="ij")
    out = np.empty((wl.batch, H, W), dtype=np.float32)
    for b in range(wl.batch):
        img = np.full((H, W), g.uniform(0.0, 1.0))
        for _ in range(discs):
            r = g.uniform(2.0, max(2.0, H / 4.0))
            cy, cx = g.uniform(0.0, H), g.uniform(0.0, W)
            level = g.uniform(0.0, 1.0)
            img[(yy - cy) ** 2 + (xx - cx) ** 2 <= r * r] = level
        img = img + g.normal(0.0, noise, size=(H, W))
        out[b] = img.astype(np.float32)
    return out


def normal(shape, seed: int, tag: str, scale: float = 1.0) -> np.ndarray:
    a = rng(seed, tag).standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a


def qkv(wl: Workload, seed: int | None = None):
    """Three fp32 arrays [U, N, heads, dh]."""
    s = wl.seed if seed is None else seed
    shape = (wl.units, wl.unit_tokens, wl.heads, wl.head_dim)
    return tuple(normal(shape, s, t, wl.qkv_scale) for t in ("q", "k", "v"))


def mlp_params(wl: Workload, seed: int | None = None, bias_scale: float = 0.0):
    """x [B, T, C], w1 [hidden, C], b1 [hidden], w2 [C, hidden], b2 [C] as fp32 arrays."""
    s = wl.seed if seed is None else seed
    x = normal((wl.batch, wl.tokens_per_image, wl.dim), s, "x")
    w1 = normal((wl.hidden, wl.dim), s, "w1", 0.02)
    w2 = normal((wl.dim, wl.hidden), s, "w2", 0.02)
    if bias_scale:
        b1 = normal((wl.hidden,), s, "b1", bias_scale)
        b2 = normal((wl.dim,), s, "b2", bias_scale)
    else:
        b1 = np.zeros((wl.hidden,), np.float32)
        b2 = np.zeros((wl.dim,), np.float32)
    return x, w1, b1, w2, b2


BLOCK_PARAM_NAMES = ("ln1_w", "ln1_b", "w_qkv", "b_qkv", "w_proj", "b_proj", "ln2_w", "ln2_b",
                     "w1", "b1", "w2", "b2")


def block_params(dim: int, hidden: int, seed: int, block: int) -> dict:
    """One encoder block's weights as fp32 arrays, keyed by BLOCK_PARAM_NAMES (Linear weights in
    the [out, in] convention; w_qkv's 3*dim rows are ordered q, k, v)."""
    shapes = {"w_qkv": (3 * dim, dim), "w_proj": (dim, dim), "w1": (hidden, dim), "w2": (dim, hidden)}
    out = {}
    for name in BLOCK_PARAM_NAMES:
        g = rng(seed, name, block)
        if name in shapes:
            shp = shapes[name]
            a = g.standard_normal(size=shp, dtype=np.float32) * np.float32(1.0 / np.sqrt(shp[1]))
        else:
            n = {"b_qkv": 3 * dim, "b1": hidden}.get(name, dim)
            a = g.standard_normal(size=(n,), dtype=np.float32) * np.float32(0.1)
            if name.endswith("_w"):
                a = a + np.float32(1.0)
        out[name] = a.astype(np.float32)
    return out


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """Round an fp32 array to bf16 (round to nearest even), as a CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 tensor (any device) to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
