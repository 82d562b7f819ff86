"""Host-side helpers for running the verification step on several GPUs.

A batch-1 step does not shard, so each GPU runs an independent replica; batched steps
shard by sequence (the sequences of a step are independent) with no collective on the
data path.  torch.distributed only supplies the barrier and the max-over-ranks timing
reduction.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def shard_sequences(batch: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) block of sequences owned by `rank`; sizes differ by <= 1."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(values: Sequence[float], dist=None, device=None) -> List[float]:
    """Element-wise maximum of `values` over all ranks (identity without a process group)."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]
