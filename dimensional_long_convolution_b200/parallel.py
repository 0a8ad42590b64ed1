"""Host-side helpers for running the convolution on several GPUs.

The (b, c) volumes of the gated convolution are independent (the pages'
operator has no exchange between volumes), so several GPUs need no data-path
collective: each rank takes a contiguous slice of the global batch and runs the
library on it.  Only timing uses a collective (the maximum over ranks).
"""
from __future__ import annotations

from typing import Tuple


def shard_range(total: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous slice [start, stop) of ``total`` units owned by ``rank``;
    the first ``total % world`` ranks take one extra unit."""
    if world < 1 or not (0 <= rank < world) or total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Maximum of a per-rank scalar (a step time) over all ranks."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
