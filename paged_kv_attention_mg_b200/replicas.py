"""Multi-GPU plumbing for the hot path: independent replicas, no data-path collective.

The attention path shards with no exchange step: (request, kv head) units are
independent ("mini-sglang from Scratch Stage 4 · Faster and bigger", §What it
prints: under tensor parallelism each rank holds its own share of the KV heads
and its own pool; the only collective, the all-reduce after o_proj, lies
outside attention).  So N GPUs run N replicas, one process per GPU, each with
its own seeded batch (weak scaling).  torch.distributed is used only to line
the ranks up around the timed region and to take the max of their times.

``shard_requests`` splits one global batch across ranks instead (the strong-
scaling alternative), as contiguous request ranges.
"""
from __future__ import annotations

import dataclasses
import datetime
import os
from typing import Optional, Tuple

import torch

RANK_SEED_STRIDE = 7919


def rank_spec(spec, rank: int):
    """The workload a rank runs: rank 0 runs the named workload itself, every
    other rank the same shapes with its own seed."""
    return dataclasses.replace(spec, seed=spec.seed + RANK_SEED_STRIDE * rank) if rank else spec


def shard_requests(batch: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [begin, end) request range of `rank`; ranges cover the batch
    exactly once and differ in size by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(batch, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


class Replicas:
    """Rank/world from the torchrun environment; a process group only when world > 1."""

    def __init__(self, want: Optional[int] = None, backend: str = "nccl", timeout_s: float = 180.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if want is not None and want != self.world:
            raise SystemExit(f"asked for {want} GPUs but WORLD_SIZE={self.world}: launch N>1 with torchrun")
        self.backend = backend
        self.pg = None
        if self.world > 1:
            import torch.distributed as dist
            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.pg = dist

    @property
    def _device(self):
        return torch.device("cuda", self.local) if self.backend == "nccl" else torch.device("cpu")

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def _reduce(self, x: float, op) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self._device)
        self.pg.all_reduce(t, op=op)
        return float(t.item())

    def max(self, x: float) -> float:
        return self._reduce(x, self.pg.ReduceOp.MAX if self.pg else None)

    def sum(self, x: float) -> float:
        return self._reduce(x, self.pg.ReduceOp.SUM if self.pg else None)

    def close(self):
        if self.pg:
            self.pg.barrier()
            self.pg.destroy_process_group()
            self.pg = None
