"""Replica ranks: one process per GPU, each running its own independent system.

REANN MD on one node shards as independent replicas (the energy+force path
has no exchange step between GPUs when every GPU owns a whole system), so the
only collectives are the host-side ones that bracket a timed region: a
barrier before and after it, the maximum of the ranks' device times and the
sum of the units they processed.  Every rank takes the same collective steps
in the same order, including when it has nothing to report.

The group is backend-neutral: NCCL needs its reduction buffers on the GPU,
gloo (the CPU test backend) on the host.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass
from typing import Callable


@dataclass
class RankInfo:
    rank: int
    world: int
    local: int

    @classmethod
    def from_env(cls) -> "RankInfo":
        return cls(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                   int(os.environ.get("LOCAL_RANK", "0")))


class RankGroup:
    """Barrier / max / sum over the ranks of an initialised process group, or
    the identity for a single process."""

    def __init__(self, dist=None, device: str = "cpu"):
        self.dist = dist
        self.device = device

    @classmethod
    def init(cls, info: RankInfo, backend: str, timeout_s: float = 300.0) -> "RankGroup":
        if info.world <= 1:
            return cls()
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
        return cls(dist, f"cuda:{info.local}" if backend == "nccl" else "cpu")

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def _reduce(self, val: float, op) -> float:
        import torch
        t = torch.tensor([float(val)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=op)
        return float(t.item())

    def max(self, val: float) -> float:
        return float(val) if self.dist is None else self._reduce(val, self.dist.ReduceOp.MAX)

    def sum(self, val: float) -> float:
        return float(val) if self.dist is None else self._reduce(val, self.dist.ReduceOp.SUM)

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()
            self.dist = None


@dataclass
class Timed:
    ms: float        # slowest rank's time of the region
    units: float     # units processed by all ranks
    result: object   # this rank's return value of the region

    @property
    def throughput(self) -> float:
        """Whole-job units per second."""
        return self.units / (self.ms * 1e-3) if self.ms > 0 else float("inf")


def timed_region(group: RankGroup, run: Callable[[], object], clock: Callable[[Callable[[], object]], tuple],
                 units: float) -> Timed:
    """Barrier, run `run` under `clock` on every rank, barrier, then reduce:
    time = max over ranks, units = sum over ranks.

    `clock(run)` returns (elapsed_ms, result); on a GPU it brackets the call
    with CUDA events on the launching stream and synchronises on both sides."""
    group.barrier()
    ms, out = clock(run)
    group.barrier()
    return Timed(group.max(ms), group.sum(units), out)


def cuda_event_clock(stream) -> Callable[[Callable[[], object]], tuple]:
    """Device time of one call: CUDA events recorded on `stream`, with a
    device synchronisation before and after."""
    import torch

    def clock(run):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        out = run()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b), out

    return clock


def host_clock(run) -> tuple:
    """Wall time of one call (CPU-only processes)."""
    import time
    t0 = time.perf_counter()
    out = run()
    return (time.perf_counter() - t0) * 1e3, out

