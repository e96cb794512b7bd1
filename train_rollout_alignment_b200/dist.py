"""Multi-GPU plumbing for the benchmark: one process per GPU, every rank works
on its own layer stack (weak scaling), and the only collective is the max of
the ranks' elapsed times.  The quantization path itself has no data-path
collective: each 16-value block depends only on its own tensor's amax.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def world() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def nccl_init_log() -> None:
    """Keep NCCL's communicator set-up log (rank count, transports, NVLS) on,
    written to stderr so that stdout carries only the result line; a caller's
    own NCCL_DEBUG settings win."""
    os.environ.setdefault("NCCL_DEBUG", "INFO")
    os.environ.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
    os.environ.setdefault("NCCL_DEBUG_FILE", "/dev/stderr")


def init(backend: str, timeout_s: float = 300.0) -> None:
    if not dist.is_initialized():
        if backend == "nccl":
            nccl_init_log()
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Max of a float over all ranks (the job's time is its slowest rank's)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world_size: int, max_seconds: float) -> float:
    """Whole-job throughput: units every rank processed / the slowest rank's time."""
    return units_per_rank * world_size / max_seconds


def finish() -> None:
    if dist.is_initialized():
        barrier()
        dist.destroy_process_group()
