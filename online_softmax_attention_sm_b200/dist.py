"""Host-side logic of multi-GPU runs: every rank runs an independent replica of the work
(units are independent; nothing is exchanged on the data path), timings are reduced with
a max over ranks, and each rank draws its own inputs."""
from __future__ import annotations

import torch
import torch.distributed as dist


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's replica: distinct per rank, equal to the base seed on rank 0."""
    return int(base_seed) + 1000 * int(rank)


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group).
    Every rank must call it in the same order."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(work_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Whole-job throughput of weak-scaled replicas: all ranks' work over the slowest rank."""
    return world * work_per_rank / slowest_seconds
