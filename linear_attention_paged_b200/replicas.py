"""Host-side plumbing for running the HSA step as independent replicas, one per GPU.

The step has no exchange between layers, denoising steps or chunks, so N ranks run
N independent problems (weak scaling) and the data path needs no collective; the
only cross-rank traffic is the barrier around the timed region and the max of the
ranks' device times.  These helpers work with any torch.distributed backend (NCCL
on GPUs; gloo on CPU in the tests)."""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist

RANK_SEED_STRIDE = 1000


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s own problem: distinct per rank, rank 0 keeps base_seed."""
    return base_seed + RANK_SEED_STRIDE * rank


def env_ranks() -> tuple[int, int, int]:
    """(rank, world, local_rank) from the launcher's environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(world: int, backend: str, timeout_s: float = 120.0, device=None) -> None:
    """Join the process group with a short timeout, so that ranks waiting for a rank
    that died end with an error instead of waiting for good."""
    if world <= 1:
        return
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(value: float, world: int, device="cpu") -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, elapsed_max_s: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * float(units_per_rank) / float(elapsed_max_s)


def shutdown(world: int) -> None:
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
