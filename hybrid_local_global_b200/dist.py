"""Process-group plumbing for running the attention path on N GPUs of one node.

The path partitions into independent units (sequences and KV-head groups of
every layer), so N GPUs run N replicas of a workload with no collective on
the data path. The only collectives are the barrier around a timed region
and one max-reduction of the per-rank device time: a multi-GPU number is the
slowest rank's time, and the whole-job rate is the units of all ranks over it.

One process per GPU, launched by torchrun (RANK / LOCAL_RANK / WORLD_SIZE /
MASTER_ADDR / MASTER_PORT in the environment); NCCL on GPUs, gloo for the
host-only tests of this module.
"""
from __future__ import annotations

import datetime
import os

import torch


class Ranks:
    """World size, rank and local rank of this process; `device` is where the
    max-reduction's scalar lives (cuda:local for NCCL, cpu for gloo)."""

    def __init__(self, world: int, rank: int, local: int, backend: str | None):
        self.world, self.rank, self.local, self.backend = world, rank, local, backend

    @property
    def device(self) -> torch.device:
        return torch.device("cuda", self.local) if self.backend == "nccl" else torch.device("cpu")

    def barrier(self) -> None:
        if self.world > 1:
            torch.distributed.barrier()

    def max_over_ranks(self, x: float) -> float:
        """The largest x over all ranks (every rank gets it)."""
        if self.world == 1:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    def close(self) -> None:
        if self.world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


def setup(backend: str = "nccl", timeout_s: int = 600) -> Ranks:
    """Join the process group described by the environment (no-op for one
    process). A short timeout makes ranks that wait on a dead peer fail."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return Ranks(world, rank, local, backend if world > 1 else None)


def whole_job_rate(units_per_rank: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job throughput of N replicas: every rank processes
    `units_per_rank` per step; the job takes the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("non-positive time")
    return world * units_per_rank * steps / (max_ms / 1e3)
