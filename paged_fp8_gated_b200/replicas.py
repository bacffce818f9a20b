"""Host-side plumbing for running the step as independent replicas, one process
per GPU (the step has no cross-GPU exchange: requests and KV heads are
independent, and the head split across GPUs is already applied to the inputs).

Ranks share nothing but a barrier around the timed region and a max-reduction
of their times; the job's throughput is the sum of the ranks' work over the
slowest rank's time (weak scaling: every rank runs a full-size step).
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def rank_info() -> tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(base_seed: int, rank: int) -> int:
    """Each replica draws its own inputs."""
    return base_seed + 1000 * rank


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device: torch.device | str = "cpu") -> float:
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / slowest_seconds
