"""Seeded synthetic workloads for the paged KV hot path.

This module only draws inputs: request lengths, slot assignment, page-table
rows, metadata and bf16 tensors.  It holds none of the attention arithmetic,
so both the CUDA path's tests/bench and the oracle can take their inputs from
it.  Everything is drawn on the CPU from ``torch.Generator('cpu')`` so a given
(workload, layer) gives the same bits on every machine.

Shapes follow the engine's own structures ("手写 mini-sglang 阶段一 · Engine 与
采样器", §初始化的顺序 and §手工驱动引擎):

* KV pool per layer: K and V, each ``[num_slots, Hkv, D]`` bf16 (page_size 1,
  so a page is a slot).  The last slot is the dummy slot that padded requests
  would write to; it is never assigned to a real request.
* page table: int32 ``[B + 1, align32(max_len)]``; row ``table_idx[r]`` holds the
  slot of every token of request r; the last row is the dummy request's and,
  like every unused entry, points at the dummy slot.
* a request has ``cached_len`` tokens already in the pool and ``seq_len`` tokens
  after this step; its new tokens' K/V go to
  ``out_loc = page_table[table_idx[r], cached_len:seq_len]``, and the new tokens
  of all requests are concatenated in request order.

Recipe (the same for every workload):

1. ``gen = Generator().manual_seed(seed)`` draws, in this order: the lengths
   (decode: ``seq_len`` by the workload's rule, ``cached_len = seq_len - 1``;
   extend: ``cached_len`` then the chunk length ``n``), ``table_idx`` =
   ``randperm(B)``, and one ``randperm(num_slots - 1)`` that is cut into
   consecutive runs of ``seq_len[r]`` slots for r = 0, 1, ...  So slots are
   distinct across all requests.
2. layer ``l`` draws from ``Generator().manual_seed(seed * 1000 + 1 + l)``, in
   this order: q, k_new, v_new, k_hist, v_hist, each fp32 N(0,1) rounded to
   bf16 (round-to-nearest-even).  k_hist/v_hist fill the slots of positions
   ``[0, cached_len)``; every other slot of the pool, including the dummy slot
   and the slots the new tokens are about to be stored in, holds bf16 NaN
   (bit pattern 0xFFFF), so a read of a slot outside the history shows up as
   NaN in the output.
3. shared-prefix workloads (a radix prefix cache hit, "Mini-SGLang" tag page,
   KV Cache post): requests come in groups of consecutive requests; after
   step 1, every member's first P page-table entries are overwritten with the
   group's first member's, so the shared tokens sit in the pool once.  The
   history (step 2) holds each slot the rows reference once, in the order of
   first reference; the members' own slots of those positions are no longer
   referenced and stay NaN.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, List, Optional

import torch

NAN_BF16_BITS = 0xFFFF  # sign 1, exponent all ones, mantissa != 0 -> NaN


def align_up_32(x: int) -> int:
    return (x + 31) // 32 * 32


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    kind: str  # "decode" or "extend"
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_slots: int
    num_layers: int
    seed: int
    max_len: int  # upper bound of seq_len by construction (page-table width before align)
    description: str
    lengths: Callable = field(repr=False, compare=False, default=None)
    share: Optional[tuple] = None  # (members per group, shared prefix length P) or None
    mixed: bool = False  # a chunked-prefill scheduler's mixed batch (served by mg_mixed_attn)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


def _fixed(values):
    def draw(gen, batch):
        seq = torch.tensor(values, dtype=torch.int64)
        return seq - 1, seq
    return draw


def _uniform_decode(lo, hi):
    def draw(gen, batch):
        seq = torch.randint(lo, hi + 1, (batch,), generator=gen, dtype=torch.int64)
        return seq - 1, seq
    return draw


def _lognormal_decode(mean, sigma, cap):
    # mean of the uncapped lognormal is exp(mu + sigma^2/2) = mean
    mu = math.log(mean) - sigma * sigma / 2.0

    def draw(gen, batch):
        z = torch.randn(batch, generator=gen, dtype=torch.float64)
        seq = torch.exp(mu + sigma * z).round().clamp(1, cap).to(torch.int64)
        return seq - 1, seq
    return draw


def _constant_decode(length):
    def draw(gen, batch):
        seq = torch.full((batch,), length, dtype=torch.int64)
        return seq - 1, seq
    return draw


def _uniform_extend(c_lo, c_hi, n_lo, n_hi):
    def draw(gen, batch):
        cached = torch.randint(c_lo, c_hi + 1, (batch,), generator=gen, dtype=torch.int64)
        n = torch.randint(n_lo, n_hi + 1, (batch,), generator=gen, dtype=torch.int64)
        return cached, cached + n
    return draw


def _prefix_decode(prefix, lo, hi):
    """Decode lengths P + U[lo, hi]: every request has its own tokens after the
    shared prefix (at least the new one)."""
    def draw(gen, batch):
        seq = prefix + torch.randint(lo, hi + 1, (batch,), generator=gen, dtype=torch.int64)
        return seq - 1, seq
    return draw


def _mixed(prefills, c_lo, c_hi, n_lo, n_hi, d_lo, d_hi):
    """A chunked-prefill scheduler's mixed batch: `prefills` prompt chunks
    (cached U[c_lo, c_hi], chunk U[n_lo, n_hi]) first, then decode requests (one
    new token after U[d_lo, d_hi] cached ones)."""
    def draw(gen, batch):
        pc = torch.randint(c_lo, c_hi + 1, (prefills,), generator=gen, dtype=torch.int64)
        pn = torch.randint(n_lo, n_hi + 1, (prefills,), generator=gen, dtype=torch.int64)
        dc = torch.randint(d_lo, d_hi + 1, (batch - prefills,), generator=gen, dtype=torch.int64)
        cached = torch.cat([pc, dc])
        return cached, cached + torch.cat([pn, torch.ones(batch - prefills, dtype=torch.int64)])
    return draw


WORKLOADS: List[WorkloadSpec] = [
    WorkloadSpec("tiny_decode", "decode", 3, 16, 8, 128, 512, 1, 1000, 12,
                 "3 requests, lengths 5/9/12 (new token included), Hq16/Hkv8, pool 512",
                 _fixed([5, 9, 12])),
    WorkloadSpec("qwen3_0.6b_decode_28l", "decode", 64, 16, 8, 128, 200_000, 28, 1001, 2048,
                 "Qwen3-0.6B attention shape, 28 layers, batch 64, lengths U[128,2048], pool 200k",
                 _uniform_decode(128, 2048)),
    WorkloadSpec("batch256_gqa4_decode", "decode", 256, 32, 8, 128, 1_200_000, 1, 1002, 4096,
                 "batch 256, GQA 4, lengths lognormal(mean 1024, sigma 1) capped at 4096, pool 1.2M",
                 _lognormal_decode(1024.0, 1.0, 4096)),
    WorkloadSpec("longctx_gqa8_decode", "decode", 8, 32, 4, 128, 300_000, 1, 1003, 32768,
                 "batch 8, every length 32768, GQA 8, pool 300k (split-KV + merge)",
                 _constant_decode(32768)),
    WorkloadSpec("chunked_prefill_extend", "extend", 16, 16, 8, 128, 100_000, 1, 1004, 3072,
                 "16 requests, cached U[0,2048], chunk U[256,1024], Hq16/Hkv8, pool 100k",
                 _uniform_extend(0, 2048, 256, 1024)),
    WorkloadSpec("shared_prefix_decode", "decode", 64, 16, 8, 128, 200_000, 1, 1005, 2560,
                 "Qwen3-0.6B attention shape, batch 64 in 8 groups of 8 sharing a 2048-token prefix, "
                 "own tokens U[16,512] after it, pool 200k",
                 _prefix_decode(2048, 16, 512), share=(8, 2048)),
    WorkloadSpec("mixed_prefill_decode", "extend", 204, 16, 8, 128, 300_000, 1, 1006, 3072,
                 "one launch over a mixed batch: 4 prompt chunks (cached U[0,1024], chunk U[256,1024]) and "
                 "200 decode requests (one new token after U[128,2047] cached), Hq16/Hkv8, pool 300k",
                 _mixed(4, 0, 1024, 256, 1024, 128, 2047), mixed=True),
]

BY_NAME = {w.name: w for w in WORKLOADS}


def custom_spec(kind: str, lengths_cached, lengths_seq, num_q_heads: int, num_kv_heads: int,
                num_slots: int, seed: int, head_dim: int = 128, name: str = "custom",
                num_layers: int = 1) -> WorkloadSpec:
    """A workload with explicit per-request (cached_len, seq_len), for tests."""
    cached = [int(c) for c in lengths_cached]
    seq = [int(s) for s in lengths_seq]

    def draw(gen, batch):
        return torch.tensor(cached, dtype=torch.int64), torch.tensor(seq, dtype=torch.int64)

    return WorkloadSpec(name, kind, len(seq), num_q_heads, num_kv_heads, head_dim, num_slots,
                        num_layers, seed, max(seq) if seq else 1, "custom", draw)


@dataclass
class Step:
    """Metadata of one batch step (shared by every layer of that step)."""
    spec: WorkloadSpec
    cached_len: torch.Tensor  # [B] int32
    seq_len: torch.Tensor  # [B] int32
    table_idx: torch.Tensor  # [B] int32
    page_table: torch.Tensor  # [B+1, stride] int32
    out_loc: torch.Tensor  # [T] int32, T = sum(seq_len - cached_len)
    q_offset: torch.Tensor  # [B+1] int32 prefix sums of new-token counts
    dummy_slot: int
    group_first: Optional[torch.Tensor] = None  # shared-prefix workloads: [G+1] int32
    prefix_len: Optional[torch.Tensor] = None   # [G] int32

    @property
    def batch(self) -> int:
        return int(self.seq_len.shape[0])

    @property
    def num_new_tokens(self) -> int:
        return int(self.out_loc.shape[0])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_len.max()) if self.batch else 0

    @property
    def max_q_len(self) -> int:
        n = self.seq_len - self.cached_len
        return int(n.max()) if self.batch else 0

    def history_slots(self) -> torch.Tensor:
        """Slots of positions [0, cached_len) of every request, request order,
        each slot once (rows that share a prefix reference its slots again)."""
        rows = []
        for r in range(self.batch):
            row = self.page_table[int(self.table_idx[r])]
            rows.append(row[: int(self.cached_len[r])])
        if not rows:
            return torch.zeros(0, dtype=torch.int64)
        slots = torch.cat(rows).to(torch.int64)
        uniq, inverse = torch.unique(slots, return_inverse=True)
        if uniq.numel() == slots.numel():
            return slots  # every slot once already (no shared prefix)
        first = torch.full((uniq.numel(),), slots.numel(), dtype=torch.int64)
        first.scatter_reduce_(0, inverse, torch.arange(slots.numel()), reduce="amin")
        return slots[torch.sort(first).values]


@dataclass
class LayerData:
    """Per-layer tensors (CPU, bf16 unless noted)."""
    q: torch.Tensor  # decode [B, Hq, D]; extend [T, Hq, D]
    k_new: torch.Tensor  # [T, Hkv, D]
    v_new: torch.Tensor  # [T, Hkv, D]
    hist_slots: torch.Tensor  # [H] int64
    k_hist: torch.Tensor  # [H, Hkv, D]
    v_hist: torch.Tensor  # [H, Hkv, D]


def make_step(spec: WorkloadSpec, page_table_stride: Optional[int] = None) -> Step:
    gen = torch.Generator().manual_seed(spec.seed)
    cached, seq = spec.lengths(gen, spec.batch)
    batch = spec.batch
    assert cached.shape == (batch,) and seq.shape == (batch,)
    assert bool((cached >= 0).all()) and bool((seq >= cached).all())
    table_idx = torch.randperm(batch, generator=gen) if batch else torch.zeros(0, dtype=torch.int64)
    dummy_slot = spec.num_slots - 1
    total = int(seq.sum())
    if total > dummy_slot:
        raise ValueError(f"{spec.name}: {total} tokens do not fit {dummy_slot} slots")
    perm = torch.randperm(dummy_slot, generator=gen)
    stride = page_table_stride or align_up_32(max(spec.max_len, int(seq.max()) if batch else 1))
    page_table = torch.full((batch + 1, stride), dummy_slot, dtype=torch.int32)
    out_loc = []
    pos = 0
    for r in range(batch):
        L = int(seq[r])
        row = int(table_idx[r])
        page_table[row, :L] = perm[pos:pos + L].to(torch.int32)
        pos += L
        out_loc.append(page_table[row, int(cached[r]):L])
    n = (seq - cached).to(torch.int64)
    q_offset = torch.zeros(batch + 1, dtype=torch.int64)
    if batch:
        q_offset[1:] = torch.cumsum(n, 0)
    step = Step(spec=spec, cached_len=cached.to(torch.int32), seq_len=seq.to(torch.int32),
                table_idx=table_idx.to(torch.int32), page_table=page_table,
                out_loc=(torch.cat(out_loc) if out_loc else torch.zeros(0, dtype=torch.int32)),
                q_offset=q_offset.to(torch.int32), dummy_slot=dummy_slot)
    if spec.share:
        share_prefixes(step, spec.share[0], spec.share[1])
    return step


def share_prefixes(step: Step, members: int, prefix: int) -> None:
    """Groups of `members` consecutive requests share their first `prefix`
    page-table entries (the first member's slots); sets group_first /
    prefix_len.  The prefix must leave every member at least its new token."""
    b = step.batch
    firsts = list(range(0, b, members)) + [b]
    plen = []
    for g0, g1 in zip(firsts[:-1], firsts[1:]):
        P = min(prefix, int(step.seq_len[g0:g1].min()) - 1, int(step.cached_len[g0:g1].min()))
        lead = int(step.table_idx[g0])
        for r in range(g0 + 1, g1):
            step.page_table[int(step.table_idx[r]), :P] = step.page_table[lead, :P]
        plen.append(P)
    step.group_first = torch.tensor(firsts, dtype=torch.int32)
    step.prefix_len = torch.tensor(plen, dtype=torch.int32)


def _bf16_normal(gen, shape) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_layer(step: Step, layer: int = 0) -> LayerData:
    spec = step.spec
    gen = torch.Generator().manual_seed(spec.seed * 1000 + 1 + layer)
    t = step.num_new_tokens
    hq, hkv, d = spec.num_q_heads, spec.num_kv_heads, spec.head_dim
    q_rows = step.batch if spec.kind == "decode" else t
    q = _bf16_normal(gen, (q_rows, hq, d))
    k_new = _bf16_normal(gen, (t, hkv, d))
    v_new = _bf16_normal(gen, (t, hkv, d))
    hist = step.history_slots()
    k_hist = _bf16_normal(gen, (hist.shape[0], hkv, d))
    v_hist = _bf16_normal(gen, (hist.shape[0], hkv, d))
    return LayerData(q=q, k_new=k_new, v_new=v_new, hist_slots=hist, k_hist=k_hist, v_hist=v_hist)


def build_pool(step: Step, hist_slots: torch.Tensor, hist: torch.Tensor,
               device: str | torch.device = "cpu") -> torch.Tensor:
    """A [num_slots, Hkv, D] bf16 pool: NaN everywhere, history rows scattered in."""
    spec = step.spec
    pool = torch.empty((spec.num_slots, spec.num_kv_heads, spec.head_dim), dtype=torch.bfloat16,
                       device=device)
    pool.view(torch.int16).fill_(-1)  # 0xFFFF == bf16 NaN
    if hist_slots.numel():
        pool.index_copy_(0, hist_slots.to(device), hist.to(device))
    return pool


def bits(t: torch.Tensor):
    """uint16 numpy view of a CPU bf16 tensor (how bf16 crosses to the oracle)."""
    import numpy as np
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
