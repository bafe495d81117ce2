"""Host-side logic of multi-GPU runs: the path has no exchange step, so N GPUs
run N independent replicas (one process per GPU), each on its own seeded
streams, and a run's time is the slowest replica's.  Nothing here touches the
data path."""
from __future__ import annotations

import torch


def replica_stream_layer(rank: int, layer: int) -> int:
    """Layer index fed to the input generator for (replica rank, layer): every
    replica gets streams of its own."""
    return layer + 1000 * rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar (time) over the process group."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds
