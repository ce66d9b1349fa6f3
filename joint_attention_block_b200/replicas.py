"""Host-side plumbing of multi-GPU runs: N independent replicas, one per rank.

The block does not shard at batch 1, so ranks exchange nothing on the data path;
the only collectives are the barrier around the timed region and the max over
ranks of the device time, from which the whole-job throughput is computed.
Works with the nccl backend (CUDA tensors) and with gloo (CPU tensors, tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world() -> int:
    return dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1


def barrier() -> None:
    if world() > 1:
        dist.barrier()


def max_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """The largest value any rank reports (all ranks get it)."""
    if world() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, ms_local: float, device: torch.device | str = "cpu"):
    """(units/s over all ranks, slowest rank's ms): every rank processed units_per_rank."""
    ms = max_over_ranks(ms_local, device)
    return units_per_rank * world() / (ms / 1e3), ms
