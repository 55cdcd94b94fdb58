"""Host plumbing for running independent streams on several GPUs, one process
per GPU. Streams are independent, so they are partitioned by rank with no
exchange on the data path (weak scaling); only the timing is reduced: the
job's time is the slowest rank's."""
from __future__ import annotations

from typing import List, Optional

import torch
import torch.distributed as dist


def rank_stream_ids(rank: int, streams_per_rank: int) -> List[int]:
    """Global ids of the streams rank `rank` holds: rank*B .. rank*B + B - 1."""
    if rank < 0 or streams_per_rank < 1:
        raise ValueError("rank must be >= 0 and streams_per_rank >= 1")
    return [rank * streams_per_rank + b for b in range(streams_per_rank)]


def max_over_ranks(value: float, device: Optional[torch.device | str] = None) -> float:
    """Max of a per-rank number over the default process group (the value
    itself when no group is initialised or the world has one rank). With
    NCCL pass a CUDA device; with gloo the CPU default serves."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, elapsed_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's elapsed time (ms)."""
    if elapsed_ms <= 0 or world < 1:
        raise ValueError("elapsed_ms must be > 0 and world >= 1")
    return units_per_rank * world / (elapsed_ms / 1000.0)
