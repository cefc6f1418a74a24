"""Host-side plumbing for running the path on several GPUs of one node.

The Orthrus round shards by sequence with no exchange step: every rank owns its
own sequences, pages and buffers and runs all kernels independently (weak
scaling). The only collectives are a barrier around the timed region and one
all-reduce of a scalar (the slowest rank's time); neither is on the data path.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_world() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 300.0) -> tuple[int, int, int]:
    """Join the process group when launched with more than one rank (and pick this
    rank's GPU for nccl). Returns (world, rank, local rank)."""
    world, rank, local = env_world()
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    elif world == 1 and backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The largest value of x over all ranks (one scalar all-reduce)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's own batch: different data per rank, reproducible."""
    return base + 1000 * rank


def shard(n: int, rank: int, world: int) -> range:
    """Contiguous share of n items for this rank (sizes differ by at most one)."""
    lo = n * rank // world
    hi = n * (rank + 1) // world
    return range(lo, hi)


def weak_scaling_throughput(units_per_rank_step: float, ms_per_step_max: float,
                            world: int) -> float:
    """Whole-job throughput: every rank processed its units in the slowest rank's time."""
    return world * units_per_rank_step / (ms_per_step_max * 1e-3)


def finish(world: int) -> None:
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
