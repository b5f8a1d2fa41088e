"""Splitting one attention call across GPUs, one process per GPU.

The attention core partitions without any exchange: a (batch, kv head) unit
together with the rep = Hq / Hkv query heads that read it is independent of
every other unit, and tile maps do not depend on the head. A rank therefore
runs the ordinary call on a contiguous range of kv heads (views of the caller's
tensors, no copies): q, gate and out keep their strides and start at the first
query head of the range; k and v start at the range's first kv head.
"""
from __future__ import annotations

from typing import List, Tuple


def kv_head_range(num_kv_heads: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous kv heads [start, stop) of `rank`; sizes differ by at most one."""
    if not (0 <= rank < world):
        raise ValueError("rank out of range")
    base, extra = divmod(num_kv_heads, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def partition(num_kv_heads: int, world: int) -> List[Tuple[int, int]]:
    return [kv_head_range(num_kv_heads, r, world) for r in range(world)]


def shard_views(q, k, v, gate, out, rank: int, world: int):
    """Views of [B, L, H, d] tensors holding this rank's kv heads and their query heads."""
    Hq, Hkv = q.shape[2], k.shape[2]
    rep = Hq // Hkv
    g0, g1 = kv_head_range(Hkv, rank, world)
    qs = slice(g0 * rep, g1 * rep)
    ks = slice(g0, g1)
    return (q[:, :, qs], k[:, :, ks], v[:, :, ks], None if gate is None else gate[:, :, qs], out[:, :, qs])
