"""Independent replicas across GPUs (one process per GPU).

The DSA hot path has no exchange step on one GPU: decode sequences and prefill
queries are independent.  Several GPUs therefore run independent replicas, each
with its own seeded batch, and meet only to time the job: a barrier on both sides
of the timed region and the maximum step time over ranks.  There is no data-path
collective.

Backend: NCCL between GPUs, gloo when the processes have no GPU (tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank_world():
    """(rank, world, local_rank) from the launcher's environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def setup(timeout_s: float = 120.0, cpu: bool = False):
    """Joins the process group when launched with WORLD_SIZE > 1; returns
    (rank, world, device).  Each rank drives the GPU of its local rank (cpu=True:
    no GPU, gloo)."""
    rank, world, local = env_rank_world()
    use_cuda = torch.cuda.is_available() and not cpu
    device = torch.device("cuda", local) if use_cuda else torch.device("cpu")
    if use_cuda:
        torch.cuda.set_device(device)
    if world > 1 and not dist.is_initialized():
        dist.init_process_group("nccl" if use_cuda else "gloo",
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world, device


def barrier(world: int, device: torch.device):
    if world > 1:
        dist.barrier()
    if device.type == "cuda":
        torch.cuda.synchronize(device)


def max_over_ranks(x: float, world: int, device: torch.device) -> float:
    """The maximum of x over all ranks (x itself for one rank)."""
    if world == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, ms_per_step_max: float, world: int) -> float:
    """Whole-job rate: every rank processes units_per_rank per step, and the job's
    step lasts as long as the slowest rank's."""
    return units_per_rank * world / (ms_per_step_max / 1e3)


def replica_seed(seed: int, rank: int) -> int:
    """A distinct, reproducible input seed per replica."""
    return seed + 1000 * rank


def teardown(world: int):
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
