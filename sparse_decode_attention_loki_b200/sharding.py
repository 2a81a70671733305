"""Multi-GPU partition of a decode step.

Every step of Loki decode attention is independent per (batch, KV head) row,
and the basis P is per KV head, so a batch splits across GPUs with no exchange
at all: each rank owns a contiguous range of batch entries, holds their cache
rows, and runs the whole step on its own GPU.  Nothing is communicated on the
data path.
"""
from __future__ import annotations

from typing import Tuple


def shard_batches(batch: int, world_size: int, rank: int) -> Tuple[int, int]:
    """Contiguous [begin, end) of the batch owned by `rank`; the first
    batch % world_size ranks take one extra entry.  Ranks beyond the batch get
    an empty range."""
    if world_size < 1 or not (0 <= rank < world_size):
        raise ValueError(f"bad rank {rank} of world {world_size}")
    if batch < 0:
        raise ValueError("batch must be >= 0")
    base, extra = divmod(batch, world_size)
    begin = rank * base + min(rank, extra)
    end = begin + base + (1 if rank < extra else 0)
    return begin, end
