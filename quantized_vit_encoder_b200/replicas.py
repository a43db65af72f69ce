"""Data-parallel helpers for running the tower on several GPUs (one process per GPU).

Images are independent in the ViT tower (block-diagonal attention, row-wise
GEMMs and norms), so a batch of images is split across ranks by whole images
and each rank runs its share with no collective on the data path.  These
helpers do the host-side bookkeeping.
"""
from __future__ import annotations


def shard_images(grids, world: int) -> list:
    """Split a list of (h, w) grids into `world` contiguous shards with balanced
    attention + GEMM work (cost ~ n^2 * 1152 + n * 30000 per image).
    Returns a list of index lists, one per rank (some may be empty)."""
    cost = [(h * w) ** 2 * 1152 + h * w * 30000 for h, w in grids]
    total = float(sum(cost))
    shards, cur, acc = [[] for _ in range(world)], 0, 0.0
    for i, c in enumerate(cost):
        # move to the next rank once this rank holds its share of the total
        if cur < world - 1 and shards[cur] and acc + c / 2 > total * (cur + 1) / world:
            cur += 1
        shards[cur].append(i)
        acc += c
    return shards


def token_ranges(grids) -> list:
    """[start, end) token range of each image in the packed order."""
    out, s = [], 0
    for h, w in grids:
        out.append((s, s + h * w))
        s += h * w
    return out


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
