"""One process per GPU: rank setup and the timing reductions of a multi-GPU run.

The decode path has no exchange step -- every (batch, head) state is
independent -- so N GPUs run N independent replicas of the per-GPU workload
(weak scaling) and only the host gathers the timings: the slowest rank's time
decides the whole job's throughput.
"""
from __future__ import annotations

import datetime
import os

import torch


def setup(timeout_s: int = 300):
    """Read RANK / LOCAL_RANK / WORLD_SIZE; join a process group when N > 1
    (NCCL with GPUs, gloo otherwise).  Returns (world, rank, local_rank, dist or None)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        if not dist.is_initialized():
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local, pg


def max_over_ranks(x: float, pg) -> float:
    """The largest value of x over all ranks (every rank gets it)."""
    if pg is None:
        return float(x)
    dev = "cuda" if (torch.cuda.is_available() and pg.get_backend() == "nccl") else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


def weak_scaling_value(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    return units_per_rank * world / seconds_max


def teardown(pg):
    if pg is not None and pg.is_initialized():
        pg.destroy_process_group()
