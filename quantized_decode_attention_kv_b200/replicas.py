"""Multi-GPU plumbing of the benchmark: one process per GPU, each running an independent replica
of the workload (its own layer's K/V and query; the path has no exchange step, so no
data-path collective). The only communication is timing: every rank contributes its device
time and the job time is the maximum over ranks ("Where This Fits in the Inference Stack",
Production Deployment: per-shard quantisation needs no communication).

Works with any torch.distributed backend: NCCL on GPUs, gloo for the CPU tests."""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_ranks() -> tuple[int, int, int]:
    """(rank, local rank, world size) from the launcher's environment (1 process by default)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, world: int, device=None, timeout_s: int = 180) -> None:
    """Join the process group when there is more than one rank (short timeout: a rank that
    never arrives ends the others' next collective with an error instead of a hang)."""
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if (backend == "nccl" and device is not None) else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(value: float, world: int, device="cpu") -> float:
    """The maximum of `value` over all ranks (every rank gets it)."""
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job rate: the units every rank processed divided by the job time (the slowest
    rank's time), i.e. weak scaling with a fixed amount of work per rank."""
    return world * units_per_rank / seconds


def replica_layer(rank: int) -> int:
    """Rank r replays layer r of the workload: distinct, deterministic inputs per rank."""
    return rank


def finish(world: int) -> None:
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
