"""Host-side helpers for running the WKV7 kernels on several GPUs of one node.

Every (b, h) head is an independent recurrence, so the data-parallel path
needs no collective on the data: each process (one per GPU) runs its own
batch shard, and the only communication is a barrier around the timed region
and one max-reduction of the measured time (the job is as slow as its slowest
rank).  Works with the "nccl" backend on GPUs and with "gloo" on CPUs (tests).
"""
from __future__ import annotations

import datetime
import os


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s batch shard (distinct per rank, stable)."""
    return base_seed + 1000 * rank


def aggregate_throughput(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / seconds_max


class Dist:
    """One process per device; RANK / WORLD_SIZE / LOCAL_RANK from the launcher."""

    def __init__(self, backend: str | None = None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None

    def init(self, timeout_s: float = 120.0):
        import torch
        import torch.distributed as dist
        backend = self.backend or ("nccl" if torch.cuda.is_available() else "gloo")
        self.backend = backend
        if backend == "nccl":
            torch.cuda.set_device(self.local)
        if self.world > 1:
            kwargs = dict(timeout=datetime.timedelta(seconds=timeout_s))
            if backend == "nccl":
                kwargs["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(backend, **kwargs)
            self.pg = dist
        return self

    def _device(self):
        import torch
        return torch.device("cuda", self.local) if self.backend == "nccl" else torch.device("cpu")

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        """Max of ``x`` over all ranks (identity for one process)."""
        if not self.pg:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=self._device())
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()
            self.pg = None
