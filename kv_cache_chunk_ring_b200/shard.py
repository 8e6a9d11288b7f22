"""Partition of the attention work across GPUs (one process per GPU).

Every head of every layer cache is an independent unit: the anchor / window
slot table is the same for all heads, and a head's attention reads only its
own Q, K and V.  Two partitions need no exchange on the data path:

* ``heads``: rank r owns a contiguous range of the heads of every layer cache,
  so one model's attention is split across the GPUs (strong scaling); each
  rank keeps its own slot table, identical on every rank because every rank
  appends the same frames.
* ``layers``: rank r owns whole layer caches (all heads), so the work per GPU
  stays fixed as GPUs are added (weak scaling).

Only the consumer of O (outside this path) would gather the heads.
"""
from __future__ import annotations

from typing import Tuple


def head_range(heads: int, world: int, rank: int) -> Tuple[int, int]:
    """Heads [h0, h1) of rank ``rank`` when ``heads`` heads are split over ``world``
    ranks: contiguous, sizes differ by at most one, the larger ranges first."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if heads < world:
        raise ValueError(f"{heads} heads cannot be split over {world} ranks")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def slice_heads(x, h0: int, h1: int):
    """Heads [h0, h1) of a token-major [tokens, heads, head_dim] tensor or array,
    contiguous (torch tensors stay on their device)."""
    part = x[:, h0:h1]
    if hasattr(part, "contiguous"):
        return part.contiguous()
    import numpy as np
    return np.ascontiguousarray(part)
