"""Process-group plumbing for running the decode workload on several GPUs.

The path shards without any exchange: every (agent, layer) view is
independent, so each rank holds whole agents and attends over them alone.  The
only collective is the host-side max of the timed durations (a multi-GPU
number is the slowest rank's).  One process per GPU, launched by torchrun;
NCCL when CUDA is present, gloo otherwise (tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def init_from_env(timeout_s: float = 120.0):
    """(rank, world, local_rank) from the torchrun environment; initialises the
    default process group when world > 1 and selects the local GPU."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def shard_agents(n_agents: int, rank: int, world: int):
    """Contiguous, balanced split of agent ids 0..n_agents-1 over ranks (for a
    fixed total, i.e. strong scaling); every agent lands on exactly one rank."""
    base, extra = divmod(n_agents, world)
    start = rank * base + min(rank, extra)
    return list(range(start, start + base + (1 if rank < extra else 0)))


def max_over_ranks(x: float) -> float:
    """Maximum of a host float over all ranks (identity without a process group)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def aggregate_throughput(units_per_rank: float, world: int, t_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / t_max


def shutdown():
    if dist.is_initialized():
        dist.destroy_process_group()
