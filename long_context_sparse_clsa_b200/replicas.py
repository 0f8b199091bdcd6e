"""Replicas across GPUs: one process per GPU, each running the whole decode step on its own
sequences.  Decode sequences are independent (the routing equation and the per-layer
equation of the picx.dev CLSA summary, Methodology > Architecture Overview, are per query
token), so the batch shards across ranks with no exchange on the data path; the only
collectives are the host-side barrier and the max-over-ranks reduction of a device-timed
figure.

Host plumbing only (no kernel runs here): process-group setup from the torchrun
environment, each rank's workload, the reduction, and the whole-job rate.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import replace


def env_ranks():
    """(rank, world size, local rank) from the torchrun environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 120):
    """Join the process group when the world has more than one rank; returns env_ranks().
    A short timeout makes a rank that never arrives end the others' collectives with an
    error instead of a hang."""
    rank, world, local = env_ranks()
    if world > 1:
        import torch.distributed as dist
        if not dist.is_initialized():
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world, local


def rank_workload(w, rank: int, world: int):
    """Each rank its own sequences: the workload with its seed advanced by the rank (the
    same shapes and value distribution, other draws)."""
    return replace(w, seed=w.seed + rank) if world > 1 else w


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest x over the ranks (every rank gets it): a step time of the job is the
    slowest rank's."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: the units every rank processed per second of the slowest rank."""
    return world * units_per_rank / (ms_per_step / 1e3)


def finish(world: int) -> None:
    """Last barrier, then leave the process group (every rank takes the same steps)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
