"""Document sharding of an index: contiguous row ranges (a list split across a
shard boundary simply has part of its rows on each side), the same centroids
on every shard, and each shard's id offset, so that st_merge_topk over the
shards' results reproduces the unsharded search exactly."""
from typing import Tuple

import torch


def shard_bounds(n: int, shards: int, g: int) -> Tuple[int, int]:
    """Rows [r0, r1) of shard g of `shards` (near-equal contiguous ranges)."""
    if not 0 <= g < shards:
        raise ValueError("shard index out of range")
    return g * n // shards, (g + 1) * n // shards


def shard_offsets(list_offsets: torch.Tensor, r0: int, r1: int) -> torch.Tensor:
    """CSR offsets of the rows [r0, r1) of an index whose lists own rows
    list_offsets[c] .. list_offsets[c+1]-1 (every list keeps its id; lists
    outside the range are empty)."""
    return (list_offsets.clamp(min=r0, max=r1) - r0).contiguous()


def shard_arrays(items, sigs, list_offsets, shards: int, g: int):
    """(items, sigs, offsets, id_offset) of shard g."""
    n = items.shape[0]
    r0, r1 = shard_bounds(n, shards, g)
    return items[r0:r1], sigs[r0:r1], shard_offsets(list_offsets, r0, r1), r0
