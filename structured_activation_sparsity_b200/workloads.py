"""Named synthetic workloads of the SparseSAM encoder-block hot path.

Each workload is one SAM encoder block as the SparseSAM pages describe it (SparseSAM README,
"Supported tasks" and "Results": SAM ViT-B/L/H at 64x64 tokens; Dutch technical summary,
"Probleemstelling": windowed blocks of fewer than 200 tokens per head). This module holds shapes
only; it computes nothing of the method.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    grid_h: int
    grid_w: int
    mode: str            # "global" or "window"
    window: int          # window side in tokens (window mode only)
    heads: int
    head_dim: int
    density: float
    dim: int             # C, the MLP input/output width
    hidden: int          # the MLP hidden width
    in_dtype: str        # dtype the workload is stated in ("fp32" or "bf16")
    qkv_scale: float     # Q/K/V ~ N(0,1) * qkv_scale
    seed: int

    # -- derived shapes (pure geometry) -------------------------------------------------------
    @property
    def mode_id(self) -> int:
        return 0 if self.mode == "global" else 1

    @property
    def tokens_per_image(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def padded_h(self) -> int:
        if self.mode == "global":
            return self.grid_h
        return -(-self.grid_h // self.window) * self.window

    @property
    def padded_w(self) -> int:
        if self.mode == "global":
            return self.grid_w
        return -(-self.grid_w // self.window) * self.window

    @property
    def windows_per_image(self) -> int:
        if self.mode == "global":
            return 1
        return (self.padded_h // self.window) * (self.padded_w // self.window)

    @property
    def units(self) -> int:
        return self.batch * self.windows_per_image

    @property
    def unit_tokens(self) -> int:
        return self.tokens_per_image if self.mode == "global" else self.window * self.window

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # 16x16 grid, one head; stated in fp32 and cast to bf16 at the library boundary.
    "tiny": Workload("tiny", 1, 16, 16, "global", 14, 1, 64, 0.4, 64, 256, "fp32", 1.0 / 8.0, 0),
    # SAM ViT-B global-attention block.
    "vitb_global": Workload("vitb_global", 1, 64, 64, "global", 14, 12, 64, 0.4, 768, 3072,
                            "bf16", 1.0, 1),
    # SAM ViT-B windowed blocks: 64x64 padded to 70x70, 25 windows of 14x14.
    "vitb_window": Workload("vitb_window", 4, 64, 64, "window", 14, 12, 64, 0.3, 768, 3072,
                            "bf16", 1.0, 2),
    # SAM ViT-H global block.
    "vith_global": Workload("vith_global", 4, 64, 64, "global", 14, 16, 80, 0.3, 1280, 5120,
                            "bf16", 1.0, 3),
    # One global block of the ViT-L stack (batch 8, dim 1024, 16x64 heads, MLP 4096).
    "vitl_global": Workload("vitl_global", 8, 64, 64, "global", 14, 16, 64, 0.4, 1024, 4096,
                            "bf16", 1.0, 4),
    # One windowed block of the ViT-L stack.
    "vitl_window": Workload("vitl_window", 8, 64, 64, "window", 14, 16, 64, 0.4, 1024, 4096,
                            "bf16", 1.0, 4),
}


def get(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}") from None


def attn_flops(units: int, n: int, heads: int, head_dim: int, kept_pairs_fraction: float) -> float:
    """4·U·N²·heads·dh·ρ: two products (QK^T and PV) of 2 flops per multiply-add."""
    return 4.0 * units * n * n * heads * head_dim * kept_pairs_fraction


def mlp_flops(rows: int, dim: int, hidden: int) -> float:
    """4·rows·C·hidden: fc1 and fc2, 2 flops per multiply-add."""
    return 4.0 * rows * dim * hidden


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["Workload", "WORKLOADS", "get", "attn_flops", "mlp_flops", "ceil_div"]
