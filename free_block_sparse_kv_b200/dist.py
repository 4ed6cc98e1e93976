"""Multi-process plumbing for the benchmark: one process per GPU, weak scaling.

Every (batch, head) of the path is independent, so ranks share nothing on the data
path: each rank runs its own copy of the workload (seeded by its rank) and the
only collectives are a barrier around the timed region and the max over ranks of
the measured time. torch.distributed provides both (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist

from . import workloads as W


def env_ranks():
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 300):
    """Join the process group named by the environment (no-op for one process)."""
    world, _, _ = env_ranks()
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if backend == "nccl" and device is not None else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world


def rank_workload(w: W.Workload, rank: int) -> W.Workload:
    """The rank's own problem: same shapes, its own seed."""
    return W.shrink(w, seed=w.seed + rank)


def barrier():
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of x over all ranks (x itself with one process)."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput in TFLOP/s: all ranks' work over the slowest rank's time."""
    return world * flops_per_rank / (ms_max / 1e3) / 1e12
