"""Sizing and algorithmic-work formulas for the paged KV hot path.

Host-side arithmetic only (no kernel math): how many bytes a KV pool holds per
token, and how many bytes / FLOPs one call of each operation must move or do
at minimum.  The roofline numbers that bench.py reports divide these by
measured kernel time.

Sources: "手写 mini-sglang 阶段一 · Engine 与采样器", §显存规划 (memory
planning: bytes per page = 2 (K and V) x head_dim x kv_heads of this rank x
page_size x dtype bytes x layers) and §练习/参考答案 (the worked example: 112 KiB
per token for Qwen3-0.6B in bf16, about 180k tokens on a 24 GB card); §初始化
的顺序 (the pool has num_pages + 1 pages, the extra one for the dummy request);
"mini-sglang from Scratch Stage 4 · Faster and bigger", §What it prints (with
TP=2 each rank's pool holds half the KV heads).
"""
from __future__ import annotations

from typing import Iterable, Sequence, Tuple


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, dtype_bytes: int,
                       tp_size: int = 1) -> int:
    """Bytes of K+V one token occupies across all layers on one rank."""
    heads = kv_heads_per_rank(num_kv_heads, tp_size)
    return 2 * num_layers * heads * head_dim * dtype_bytes


def kv_heads_per_rank(num_kv_heads: int, tp_size: int) -> int:
    """KV heads a tensor-parallel rank holds (replicated when heads < ranks)."""
    if num_kv_heads >= tp_size:
        if num_kv_heads % tp_size:
            raise ValueError("num_kv_heads must divide evenly across ranks")
        return num_kv_heads // tp_size
    if tp_size % num_kv_heads:
        raise ValueError("ranks must be a multiple of num_kv_heads to replicate")
    return 1


def kv_pool_shape(num_pages: int, page_size: int, num_kv_heads: int, head_dim: int,
                  tp_size: int = 1) -> Tuple[int, int, int, int]:
    """Per-layer K (or V) pool shape: one extra page for the dummy request."""
    return (num_pages + 1, page_size, kv_heads_per_rank(num_kv_heads, tp_size), head_dim)


def kv_capacity_tokens(free_bytes: float, model_bytes: float, memory_ratio: float,
                       bytes_per_token: int) -> int:
    """Tokens the pool can hold: (ratio x free memory - model) / bytes per token."""
    return int((memory_ratio * free_bytes - model_bytes) // bytes_per_token)


def store_bytes(num_tokens: int, num_kv_heads: int, head_dim: int, dtype_bytes: int = 2) -> int:
    """KV store: read k and v of the new tokens, write them to the pool, read out_loc."""
    row = num_kv_heads * head_dim * dtype_bytes
    return 2 * 2 * num_tokens * row + 4 * num_tokens


def decode_bytes(seq_lens: Iterable[int], num_q_heads: int, num_kv_heads: int, head_dim: int,
                 dtype_bytes: int = 2) -> int:
    """Decode: each (token, kv head) row of K and V read once for its GQA group,
    q read and out written once, one int32 page-table entry per token.  Split
    partials are implementation overhead and are not counted."""
    seq_lens = [int(x) for x in seq_lens]
    total = sum(seq_lens)
    batch = len(seq_lens)
    kv = total * num_kv_heads * head_dim * dtype_bytes * 2
    qo = 2 * batch * num_q_heads * head_dim * dtype_bytes
    return kv + qo + 4 * total


def decode_bytes_shared_prefix(seq_lens: Sequence[int], group_first: Sequence[int], prefix_len: Sequence[int],
                               num_q_heads: int, num_kv_heads: int, head_dim: int, dtype_bytes: int = 2) -> int:
    """Decode where groups of requests share a prefix of their page-table rows:
    the shared K/V rows (and their page-table entries) counted once per group,
    each request's own keys after the prefix once, q read and out written once."""
    seq_lens = [int(x) for x in seq_lens]
    keys = sum(seq_lens)
    for g0, g1, P in zip(group_first[:-1], group_first[1:], prefix_len):
        keys -= (int(g1) - int(g0) - 1) * int(P)  # every member but the first reads the prefix through it
    kv = keys * num_kv_heads * head_dim * dtype_bytes * 2
    qo = 2 * len(seq_lens) * num_q_heads * head_dim * dtype_bytes
    return kv + qo + 4 * keys


def extend_bytes(cached: Sequence[int], seq: Sequence[int], num_q_heads: int, num_kv_heads: int,
                 head_dim: int, dtype_bytes: int = 2) -> int:
    """Extend: every context row of K and V once, q read and out written once."""
    total_ctx = sum(int(s) for s in seq)
    total_q = sum(int(s) - int(c) for c, s in zip(cached, seq))
    kv = total_ctx * num_kv_heads * head_dim * dtype_bytes * 2
    qo = 2 * total_q * num_q_heads * head_dim * dtype_bytes
    return kv + qo + 4 * total_ctx


def extend_flops(cached: Sequence[int], seq: Sequence[int], num_q_heads: int,
                 head_dim: int) -> int:
    """Extend: QK^T and PV over the unmasked (query, key) pairs only.
    Query i of request r sees c_r + i + 1 keys, so the pairs are
    n c + n (n + 1) / 2; each pair costs 2 D (QK) + 2 D (PV) flops per q head."""
    pairs = 0
    for c, s in zip(cached, seq):
        c, n = int(c), int(s) - int(c)
        pairs += n * c + n * (n + 1) // 2
    return 4 * head_dim * num_q_heads * pairs
