"""Multi-GPU plumbing for the benchmark: one process per GPU, weak scaling.

Every (sequence, head) recurrence of the gated delta rule is independent of
every other one, so a job of `world` GPUs is `world` disjoint shards of
sequences with no data exchange at all: rank r owns the sequences of its own
synthetic batch (drawn with seed `base_seed + r`). The only collectives are
for timing: a barrier around the timed region and the maximum of the per-rank
times, so the whole-job rate is (tokens on all ranks) / (slowest rank's time).

The functions work with any torch.distributed backend (NCCL on the GPUs, gloo
on the CPU for tests); with world == 1 they make no collective call.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world_and_rank() -> tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(), dist.get_rank()
    return 1, 0


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s shard: distinct sequences on every rank."""
    return base_seed + rank


def barrier() -> None:
    world, _ = world_and_rank()
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, device: torch.device | None = None) -> float:
    """Largest value of `x` over all ranks (the job's time is its slowest rank's)."""
    world, _ = world_and_rank()
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, ms_slowest: float, world: int) -> float:
    """Whole-job throughput in units per second: every rank processes
    `units_per_rank` units, and the job ends with its slowest rank."""
    if ms_slowest <= 0:
        raise ValueError("ms_slowest must be positive")
    return world * units_per_rank / (ms_slowest * 1e-3)
