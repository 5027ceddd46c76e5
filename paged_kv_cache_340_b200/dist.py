"""Multi-GPU plumbing for the decode benchmark: one process per GPU.

Sequences are independent, so each rank runs its own batch on its own GPU
(weak scaling) and the data path has no collective. torch.distributed only
carries the barriers around the timed region and the max over ranks of the
measured time. The helpers work with NCCL (GPU) and gloo (CPU tests).
"""
from __future__ import annotations

import datetime
import os
from dataclasses import replace

import torch


def env_ranks():
    """(world, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 120):
    """Initialises the process group when WORLD_SIZE > 1 and pins the rank's GPU."""
    world, rank, local = env_ranks()
    if backend == "nccl" and torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world > 1 and not torch.distributed.is_initialized():
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def _device():
    if torch.distributed.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def barrier(world: int) -> None:
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest value any rank holds (the job's time is its slowest rank's)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_spec(spec, rank: int):
    """The workload a rank runs: same shapes, its own seed."""
    return spec if rank == 0 else replace(spec, seed=spec.seed + 1000 * rank)


def job_throughput(bytes_per_rank: int, ms_max: float, world: int) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank / (ms_max * 1e-3) / 1e9


def finalize(world: int) -> None:
    if world > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
