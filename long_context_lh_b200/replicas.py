"""Host side of a multi-GPU run: one process per GPU, each an independent
replica of the workload.

The units of the path (batch x head) are independent, so N GPUs process N
batches with no collective on the data path (weak scaling).  Only the timing
is combined across ranks: the step time of the job is the maximum over ranks
of each rank's device-timed step, and the job's throughput is the units all
ranks processed divided by that time.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class Ranks:
    rank: int
    world: int
    local_rank: int

    @property
    def multi(self) -> bool:
        return self.world > 1


def from_env(env=None) -> Ranks:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torch.distributed.run (defaults: one process)."""
    env = os.environ if env is None else env
    r = Ranks(int(env.get("RANK", "0")), int(env.get("WORLD_SIZE", "1")),
              int(env.get("LOCAL_RANK", "0")))
    if not (0 <= r.rank < r.world) or r.local_rank < 0:
        raise ValueError(f"inconsistent rank variables: {r}")
    return r


def init(ranks: Ranks, backend: str, timeout_s: float = 300.0, device=None) -> None:
    """Join the process group (no-op for one process).  A short timeout makes a
    rank that never arrives end the others' collectives with an error."""
    if not ranks.multi:
        return
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, rank=ranks.rank, world_size=ranks.world, **kw)


def finish(ranks: Ranks) -> None:
    if ranks.multi and dist.is_initialized():
        dist.destroy_process_group()


def barrier(ranks: Ranks) -> None:
    if ranks.multi:
        dist.barrier()


def max_over_ranks(ranks: Ranks, value: float, device=None) -> float:
    """The largest of the ranks' values, on every rank (identity for one process)."""
    if not ranks.multi:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Units all ranks processed per second of the slowest rank."""
    if seconds <= 0:
        raise ValueError("non-positive step time")
    return world * units_per_rank / seconds
