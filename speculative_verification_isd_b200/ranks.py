"""One process per GPU: rank set-up and the few host-side reductions the
benchmark needs.

Requests advance independently, so the step shards by batches: every rank
runs its own batch of B requests with no collective on the data path (weak
scaling).  Collectives appear only around the timed region: a barrier before
and after it, the maximum of the ranks' times, and the sum of the units they
processed.  The backend is NCCL with CUDA tensors on GPUs and gloo with CPU
tensors elsewhere (the multi-rank tests run that way).
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Ranks:
    world: int
    rank: int
    local: int
    device: torch.device

    def barrier(self) -> None:
        if self.world > 1:
            dist.barrier()

    def _reduce(self, x: float, op) -> float:
        if self.world == 1:
            return float(x)
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=op)
        return float(t.item())

    def max(self, x: float) -> float:
        """Maximum over ranks (timings: the job ends with its slowest rank)."""
        return self._reduce(x, dist.ReduceOp.MAX)

    def sum(self, x: float) -> float:
        """Sum over ranks (units processed by the whole job)."""
        return self._reduce(x, dist.ReduceOp.SUM)

    def close(self) -> None:
        if self.world > 1 and dist.is_initialized():
            dist.destroy_process_group()


def setup(use_cuda: bool = True, timeout_s: float = 120.0) -> Ranks:
    """Read RANK / LOCAL_RANK / WORLD_SIZE (torchrun's variables); for more
    than one rank, join the process group (NCCL on the local GPU, or gloo on
    the CPU) with a short timeout so that a missing rank ends in an error."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if use_cuda:
        torch.cuda.set_device(local if world > 1 else 0)
        device = torch.device("cuda", local if world > 1 else 0)
    else:
        device = torch.device("cpu")
    if world > 1:
        kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
        if use_cuda:
            dist.init_process_group("nccl", device_id=device, **kw)
        else:
            dist.init_process_group("gloo", **kw)
    return Ranks(world, rank, local, device)


def job_throughput(units_per_rank: float, ranks: Ranks, t_ms_max: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's
    time (milliseconds, already reduced with Ranks.max)."""
    return ranks.sum(units_per_rank) / (t_ms_max / 1e3)


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's batch: the ranks' synthetic batches are independent."""
    return base + rank
