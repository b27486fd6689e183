"""Rank bookkeeping of the multi-GPU benchmark.

The layer has no exchange between GPUs (the pages' expert parallelism is out of
this single-GPU path), so N GPUs run N independent replicas: one process per
GPU, launched by torch.distributed.run, each timing its own copy of the work.
The job's time is the slowest rank's, and its throughput is the units of all
ranks over that time.  The process group carries only the barrier around the
timed region and that maximum (backend "nccl" on GPUs; "gloo" for the CPU tests
of this module).
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist


@dataclass
class Ranks:
    rank: int
    world: int
    local: int

    @property
    def leader(self) -> bool:
        return self.rank == 0


def from_env() -> Ranks:
    """Rank, world size and local rank from the launcher's environment."""
    return Ranks(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                 int(os.environ.get("LOCAL_RANK", "0")))


def init(r: Ranks, backend: str, device: Optional[torch.device] = None, timeout_s: float = 120.0) -> bool:
    """Join the process group when there is more than one rank (short timeout:
    a rank that never arrives ends the others' next collective with an error)."""
    if r.world <= 1:
        return False
    kw = {"device_id": device} if (device is not None and backend == "nccl") else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return True


def barrier() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device: torch.device) -> float:
    """The largest `value` of all ranks (every rank gets it)."""
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Units of all ranks per second of the slowest rank (weak scaling)."""
    return world * units_per_rank / seconds if seconds > 0 else 0.0


def finish() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
