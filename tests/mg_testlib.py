"""Shared test helpers: tiny seeded cases and dense (non-paged) references.

The dense references gather each request's K/V rows into contiguous tensors
and call torch's fp64 ``scaled_dot_product_attention`` on the CPU, a library
routine with no paging in it.  They pin the oracle; they are never used as
the expected value for the CUDA path (the oracle is).
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

from paged_kv_attention_mg_b200 import workload as wl


class Case:
    """A seeded step with host pools that already hold the new tokens."""

    def __init__(self, spec, layer=0):
        self.spec = spec
        self.step = wl.make_step(spec)
        self.data = wl.make_layer(self.step, layer)
        self.k_pool = wl.build_pool(self.step, self.data.hist_slots, self.data.k_hist)
        self.v_pool = wl.build_pool(self.step, self.data.hist_slots, self.data.v_hist)
        # pools before the store, for store tests
        self.k_pool_before = self.k_pool.clone()
        self.v_pool_before = self.v_pool.clone()
        out_loc = self.step.out_loc.to(torch.int64)
        if out_loc.numel():
            self.k_pool.index_copy_(0, out_loc, self.data.k_new)
            self.v_pool.index_copy_(0, out_loc, self.data.v_new)

    # numpy views in the oracle's calling convention
    def oracle_args(self):
        s = self.step
        return dict(q=wl.bits(self.data.q), k_pool=wl.bits(self.k_pool), v_pool=wl.bits(self.v_pool),
                    page_table=s.page_table.numpy(), table_idx=s.table_idx.numpy(),
                    seq_len=s.seq_len.numpy())


def decode_case(lengths, hq, hkv, seed, d=128, num_slots=None):
    lengths = list(lengths)
    num_slots = num_slots or (sum(lengths) + 17)
    spec = wl.custom_spec("decode", [L - 1 for L in lengths], lengths, hq, hkv, num_slots, seed,
                          head_dim=d)
    return Case(spec)


def extend_case(cached, seq, hq, hkv, seed, d=128, num_slots=None):
    num_slots = num_slots or (sum(seq) + 23)
    spec = wl.custom_spec("extend", cached, seq, hq, hkv, num_slots, seed, head_dim=d)
    return Case(spec)


def _gather(pool, page_table, row, upto):
    slots = page_table[row, :upto].to(torch.int64)
    return pool[slots].to(torch.float64)  # [L, Hkv, D]


def dense_decode(q, k_pool, v_pool, page_table, table_idx, seq_len, scale):
    """[B, Hq, D] fp64 via SDPA on gathered contiguous K/V (GQA by repeat_interleave)."""
    b, hq, d = q.shape
    hkv = k_pool.shape[1]
    g = hq // hkv
    out = torch.empty((b, hq, d), dtype=torch.float64)
    for r in range(b):
        L = int(seq_len[r])
        row = int(table_idx[r])
        k = _gather(k_pool, page_table, row, L).repeat_interleave(g, dim=1)  # [L, Hq, D]
        v = _gather(v_pool, page_table, row, L).repeat_interleave(g, dim=1)
        qq = q[r].to(torch.float64).unsqueeze(1)  # [Hq, 1, D]
        o = F.scaled_dot_product_attention(qq, k.transpose(0, 1), v.transpose(0, 1), scale=scale)
        out[r] = o[:, 0, :]
    return out


def dense_extend(q, k_pool, v_pool, page_table, table_idx, cached_len, seq_len, q_offset, scale):
    """[T, Hq, D] fp64 via SDPA with an explicit causal mask key j <= c + i."""
    t, hq, d = q.shape
    hkv = k_pool.shape[1]
    g = hq // hkv
    out = torch.full((t, hq, d), float("nan"), dtype=torch.float64)
    for r in range(seq_len.shape[0]):
        c, L = int(cached_len[r]), int(seq_len[r])
        n = L - c
        if n == 0:
            continue
        row = int(table_idx[r])
        k = _gather(k_pool, page_table, row, L).repeat_interleave(g, dim=1).transpose(0, 1)
        v = _gather(v_pool, page_table, row, L).repeat_interleave(g, dim=1).transpose(0, 1)
        o0 = int(q_offset[r])
        qq = q[o0:o0 + n].to(torch.float64).transpose(0, 1)  # [Hq, n, D]
        i = torch.arange(n).unsqueeze(1)
        j = torch.arange(L).unsqueeze(0)
        mask = j <= c + i  # True = attend
        o = F.scaled_dot_product_attention(qq, k, v, attn_mask=mask, scale=scale)
        out[o0:o0 + n] = o.transpose(0, 1)
    return out


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()
