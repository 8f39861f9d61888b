"""Host-side plumbing of the multi-GPU benchmark: one process per GPU, each
running its own independent problem (the (batch, group) units of the method
share nothing, so the work is sharded with no collective on the data path).

torch.distributed is used only for the barrier around the timed region and
for taking the maximum of the ranks' device times.  Everything here works
with the ``gloo`` backend on CPU as well as ``nccl`` on GPUs.
"""
from __future__ import annotations

import os
from datetime import timedelta

import torch
import torch.distributed as dist


def env_ranks():
    """(world, rank, local_rank) from the launcher's environment (1, 0, 0 without one)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(world: int, backend: str, timeout_s: float = 120.0) -> None:
    """Join the process group when there is more than one rank (short timeout,
    so ranks that wait for one another fail with an error instead of hanging)."""
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s))


def finish(world: int) -> None:
    if world > 1 and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s independent problem (distinct per rank, rank 0 = base)."""
    return base_seed + 100 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The maximum of `value` over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over `steps` steps
    divided by the slowest rank's time for them (ms)."""
    if max_ms <= 0.0:
        raise ValueError("non-positive time")
    return world * units_per_rank * steps / (max_ms / 1e3)
