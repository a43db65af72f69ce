"""Seeded synthetic inputs for the FP8 ViT tower (both the CUDA path and its checker use these).

This module only draws random numbers and names shapes: it holds none of the
method's arithmetic (no quantisation, no normalisation, no rotary tables, no
patch ordering).  Everything is generated on the CPU with ``torch.Generator``
so the same seed gives the same tensors on any machine.

Dimensions follow the Qwen3-VL vision tower as described on the pages
("Qwen3-VL-8B on RTX 5090", section 3 "Inference architecture", and the
``VisionEncoder`` struct of ``spark_model/layers/vision_encoder.rs``):
hidden 1152, 16 heads x head_dim 72, MLP 4304, out_hidden 2048, 27 blocks,
DeepStack taps after blocks 8, 16, 24 and 27.

Distributions (the workloads' own recipe): x ~ N(0, s^2) with a per-image
scale s; weights ~ N(0, 0.02); biases ~ N(0, 0.01); LayerNorm gamma =
1 + N(0, 0.02), beta ~ N(0, 0.01).  Values are drawn in fp32 and rounded once
to bf16 by torch's round-to-nearest-even cast.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

HIDDEN = 1152
HEADS = 16
HEAD_DIM = 72
MLP = 4304
QKV = 3 * HIDDEN
MERGE_IN = 4 * HIDDEN          # 2x2 spatial merge concatenates 4 patches
OUT_HIDDEN = 2048
N_BLOCKS = 27
TAP_AFTER = (8, 16, 24, 27)    # 1-indexed blocks whose output feeds a merger
LN_EPS = 1e-6
ROPE_THETA = 10000.0

W_STD = 0.02
B_STD = 0.01
GAMMA_STD = 0.02


@dataclass(frozen=True)
class Workload:
    """One named input configuration."""

    name: str
    grids: tuple            # ((h, w), ...) patch grid per packed image
    n_blocks: int           # 1 for a single block, 27 for the tower
    mergers: bool           # run the four 2x2 mergers at the taps
    scales: tuple = ()      # per-image input std (default 1.0 each)
    seed_base: int = 0

    @property
    def n_tokens(self) -> int:
        return sum(h * w for h, w in self.grids)

    @property
    def input_scales(self) -> tuple:
        return self.scales if self.scales else tuple(1.0 for _ in self.grids)


# The five workloads.  The packed batch's first image is 54x18 (972 patches,
# the same count as the single 36x27 image) because the 2x2 merger needs an
# even grid on both sides.
WORKLOADS = {
    "block_16x16": Workload("block_16x16", ((16, 16),), 1, False, seed_base=0),
    "block_36x27": Workload("block_36x27", ((36, 27),), 1, False, seed_base=1000),
    "block_46x136": Workload("block_46x136", ((46, 136),), 1, False, seed_base=2000),
    "tower_46x136": Workload("tower_46x136", ((46, 136),), N_BLOCKS, True, seed_base=3000),
    "tower_packed4": Workload(
        "tower_packed4", ((54, 18), (46, 136), (24, 38), (32, 32)), N_BLOCKS, True,
        scales=(0.1, 1.0, 10.0, 1.0), seed_base=4000),
}


def _normal(g: torch.Generator, shape, std: float, mean: float = 0.0) -> torch.Tensor:
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std + mean).to(torch.bfloat16)


def block_params(seed: int) -> dict:
    """bf16 weights of one ViT block (row-major [out, in] linear weights)."""
    g = torch.Generator().manual_seed(seed)
    return {
        "norm1_w": _normal(g, (HIDDEN,), GAMMA_STD, 1.0),
        "norm1_b": _normal(g, (HIDDEN,), B_STD),
        "qkv_w": _normal(g, (QKV, HIDDEN), W_STD),
        "qkv_b": _normal(g, (QKV,), B_STD),
        "proj_w": _normal(g, (HIDDEN, HIDDEN), W_STD),
        "proj_b": _normal(g, (HIDDEN,), B_STD),
        "norm2_w": _normal(g, (HIDDEN,), GAMMA_STD, 1.0),
        "norm2_b": _normal(g, (HIDDEN,), B_STD),
        "fc1_w": _normal(g, (MLP, HIDDEN), W_STD),
        "fc1_b": _normal(g, (MLP,), B_STD),
        "fc2_w": _normal(g, (HIDDEN, MLP), W_STD),
        "fc2_b": _normal(g, (HIDDEN,), B_STD),
    }


def merger_params(seed: int) -> dict:
    """bf16 weights of one 2x2 patch merger (LayerNorm over 4608, fc1, fc2)."""
    g = torch.Generator().manual_seed(seed)
    return {
        "norm_w": _normal(g, (MERGE_IN,), GAMMA_STD, 1.0),
        "norm_b": _normal(g, (MERGE_IN,), B_STD),
        "fc1_w": _normal(g, (MERGE_IN, MERGE_IN), W_STD),
        "fc1_b": _normal(g, (MERGE_IN,), B_STD),
        "fc2_w": _normal(g, (OUT_HIDDEN, MERGE_IN), W_STD),
        "fc2_b": _normal(g, (OUT_HIDDEN,), B_STD),
    }


PATCH_DIM, POS_GRID = 1536, 48


def patch_params(seed: int) -> dict:
    """bf16 patch-embedding weights [1152, 1536], bias, and the 48 x 48 position table [2304, 1152]."""
    g = torch.Generator().manual_seed(seed)
    return {
        "w": _normal(g, (HIDDEN, PATCH_DIM), W_STD),
        "b": _normal(g, (HIDDEN,), B_STD),
        "pos": _normal(g, (POS_GRID * POS_GRID, HIDDEN), W_STD),
    }


def block_seed(wl: Workload, b: int) -> int:
    """Seed of block b (0-indexed) of a workload."""
    return wl.seed_base + 1 + b


def merger_seed(wl: Workload, t: int) -> int:
    """Seed of merger t (0..3) of a workload."""
    return wl.seed_base + 100 + t


def make_input(wl: Workload) -> torch.Tensor:
    """Packed patch embeddings [n_tokens, 1152] bf16, image i scaled by its std."""
    g = torch.Generator().manual_seed(wl.seed_base)
    parts = []
    for (h, w), s in zip(wl.grids, wl.input_scales):
        parts.append(torch.randn((h * w, HIDDEN), generator=g, dtype=torch.float32) * s)
    return torch.cat(parts, 0).to(torch.bfloat16)


def random_bf16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """Generic seeded N(0, std^2) bf16 tensor for stage-level tests."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)


def random_cu_seqlens(lengths) -> list:
    """Prefix offsets of packed segments with the given lengths (plain bookkeeping)."""
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return out
