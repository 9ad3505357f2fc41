"""Head partition of one attention layer across ranks (one process per GPU).

Every (batch, head) slice of a LiteAttention layer is independent: its Skip-Mask rows, its QK-Skip
scan and its output depend only on that slice's q, k and v. A layer therefore splits across GPUs
by heads with no exchange on the data path: rank r keeps heads [h0, h1) of every batch entry, its
own Skip-Mask rows [B, h1 - h0, T, W] from step to step, and writes o and lse for those heads
only. This module holds the bookkeeping of that split (pure host logic, no arithmetic of the
method).
"""

from __future__ import annotations

from typing import Tuple


def head_range(H: int, rank: int, world: int) -> Tuple[int, int]:
    """Heads [h0, h1) that `rank` of `world` owns. H must split evenly, so every rank carries the
    same share of the layer (H = 40 gives 40, 20, 10, 8 or 5 heads at 1, 2, 4, 5 or 8 ranks)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    per = H // world
    return rank * per, (rank + 1) * per


def shard_heads(x, rank: int, world: int, dim: int):
    """The rank's heads of a tensor whose head axis is `dim` ([B, N, H, d]: dim 2; lse [B, H, N] and
    masks [B, H, T, W]: dim 1), as a contiguous tensor (the tensor itself when world == 1)."""
    if world == 1:
        return x
    h0, h1 = head_range(x.shape[dim], rank, world)
    return x.narrow(dim, h0, h1 - h0).contiguous()
