"""Multi-GPU plumbing for the hot path: independent replicas, no data-path collective.

The attention path shards with no exchange step: (request, kv head) units are
independent ("mini-sglang from Scratch Stage 4 · Faster and bigger", §What it
prints: under tensor parallelism each rank holds its own share of the KV heads
and its own pool; the only collective, the all-reduce after o_proj, lies
outside attention).  So N GPUs run N replicas, one process per GPU, each with
its own seeded batch (weak scaling).  torch.distributed is used only to line
the ranks up around the timed region and to take the max of their times.

``shard_requests`` splits one global batch across ranks instead (the strong-
scaling alternative), as contiguous request ranges.  ``shard_kv_heads`` is the
tensor-parallel split of the same page: each rank holds a contiguous range of
KV heads with their query heads and its own pool of those heads, and runs the
unchanged kernels on them (``take_heads`` cuts a rank's slice out of a full
tensor); with fewer KV heads than ranks a head is replicated and its query
heads are divided among the ranks that hold it.
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


def shard_kv_heads(num_q_heads: int, num_kv_heads: int, rank: int, world: int) -> Tuple[int, int, int, int]:
    """KV heads [kv0, kv1) and query heads [q0, q1) of tensor-parallel `rank`.

    Query head h reads KV head h // g (g = num_q_heads // num_kv_heads), so a
    rank's query heads are those of its KV heads and the local mapping is the
    same formula on the slice.  world <= num_kv_heads: num_kv_heads / world KV
    heads per rank.  world > num_kv_heads: every KV head on world / num_kv_heads
    ranks, each with an equal share of its g query heads."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    if num_kv_heads <= 0 or num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    g = num_q_heads // num_kv_heads
    if world <= num_kv_heads:
        if num_kv_heads % world:
            raise ValueError("num_kv_heads must divide evenly across ranks")
        per = num_kv_heads // world
        kv0 = rank * per
        return kv0, kv0 + per, kv0 * g, (kv0 + per) * g
    if world % num_kv_heads:
        raise ValueError("ranks must be a multiple of num_kv_heads to replicate")
    rep = world // num_kv_heads
    if g % rep:
        raise ValueError("each KV head's query heads must divide evenly across its replicas")
    kv0 = rank // rep
    q0 = kv0 * g + (rank % rep) * (g // rep)
    return kv0, kv0 + 1, q0, q0 + g // rep


def take_heads(x: torch.Tensor, h0: int, h1: int) -> torch.Tensor:
    """Heads [h0, h1) of a [..., heads, head_dim] tensor, contiguous (a rank's
    own q / k_new / v_new rows, or its pool shard)."""
    return x[..., h0:h1, :].contiguous()


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

    def min(self, x: float) -> float:
        return -self._reduce(-x, self.pg.ReduceOp.MAX if self.pg else None)

    def close(self):
        if self.pg:
            self.pg.barrier()
            self.pg.destroy_process_group()
            self.pg = None
