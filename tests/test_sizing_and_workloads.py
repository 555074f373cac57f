"""Host logic: the sizing formulas against the pages' worked examples
(tests/golden/*.json), and the seeded workload generator's structure."""
import json
import math
import os

import numpy as np
import pytest
import torch

from paged_kv_attention_mg_b200 import roofline as rf
from paged_kv_attention_mg_b200 import workload as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_kv_bytes_per_token_worked_example():
    g = _golden("kv_sizing.json")
    got = rf.kv_bytes_per_token(g["num_layers"], g["num_kv_heads"], g["head_dim"], g["dtype_bytes"])
    assert got == g["kv_bytes_per_token"] == 112 * 1024


def test_kv_capacity_worked_example():
    g = _golden("kv_sizing.json")
    bpt = g["kv_bytes_per_token"]
    tokens = rf.kv_capacity_tokens(g["card_gb"] * 1e9, g["model_gb"] * 1e9, g["memory_ratio"], bpt)
    assert abs(g["memory_ratio"] * g["card_gb"] - g["model_gb"] - g["available_gb"]) < 1e-9
    assert abs(tokens - g["approx_capacity_tokens"]) <= g["approx_capacity_rel_tol"] * g["approx_capacity_tokens"]


def test_kv_pool_shape_with_dummy_page_and_tp():
    g = _golden("kv_pool_shape.json")
    for c in g["cases"]:
        shape = rf.kv_pool_shape(g["num_pages"], g["page_size"], g["num_kv_heads"], g["head_dim"],
                                 c["tp_size"])
        assert list(shape) == c["shape"]


def test_kv_heads_replicate_when_fewer_than_ranks():
    assert rf.kv_heads_per_rank(8, 16) == 1
    with pytest.raises(ValueError):
        rf.kv_heads_per_rank(8, 3)


def test_extend_flops_counts_unmasked_pairs():
    # brute-force count of (query, key) pairs with key <= c + i
    cached, seq = [0, 3, 7], [4, 5, 20]
    pairs = sum(1 for c, s in zip(cached, seq) for i in range(s - c) for j in range(s) if j <= c + i)
    assert rf.extend_flops(cached, seq, 16, 128) == 4 * 128 * 16 * pairs


def test_decode_bytes_formula():
    got = rf.decode_bytes([5, 9, 12], 16, 8, 128)
    assert got == 26 * 8 * 128 * 2 * 2 + 2 * 3 * 16 * 128 * 2 + 26 * 4


@pytest.mark.parametrize("spec", wl.WORKLOADS, ids=lambda s: s.name)
def test_workload_metadata_structure(spec):
    step = wl.make_step(spec)
    B = spec.batch
    assert step.page_table.shape == (B + 1, wl.align_up_32(spec.max_len))
    assert sorted(step.table_idx.tolist()) == list(range(B))
    seq, cached = step.seq_len.long(), step.cached_len.long()
    assert bool((seq >= 1).all()) and bool((seq <= spec.max_len).all())
    assert bool((cached >= 0).all()) and bool((cached < seq).all())
    if spec.kind == "decode":
        assert bool((cached == seq - 1).all())
    # slots distinct across all requests (a shared prefix counted once), never the dummy slot
    used = torch.cat([step.page_table[int(step.table_idx[r]), :int(seq[r])] for r in range(B)])
    shared = 0
    if spec.share:
        gf, pl = step.group_first.tolist(), step.prefix_len.tolist()
        assert gf[0] == 0 and gf[-1] == B and len(pl) == len(gf) - 1
        for g0, g1, P in zip(gf[:-1], gf[1:], pl):
            assert 0 < P <= int(cached[g0:g1].min())  # each member keeps at least its new token
            lead = step.page_table[int(step.table_idx[g0]), :P]
            for r in range(g0 + 1, g1):
                assert torch.equal(step.page_table[int(step.table_idx[r]), :P], lead)
            shared += (g1 - g0 - 1) * P
        assert len(step.history_slots().unique()) == step.history_slots().numel()
    assert used.unique().numel() == used.numel() - shared == int(seq.sum()) - shared
    assert int(used.max()) < step.dummy_slot == spec.num_slots - 1
    assert bool((step.page_table[B] == step.dummy_slot).all())
    # out_loc = page_table[table_idx, cached:seq], concatenated in request order
    expect = torch.cat([step.page_table[int(step.table_idx[r]), int(cached[r]):int(seq[r])]
                        for r in range(B)])
    assert torch.equal(step.out_loc, expect)
    assert step.q_offset[0] == 0 and int(step.q_offset[-1]) == step.num_new_tokens
    assert torch.equal(step.q_offset[1:] - step.q_offset[:-1], (seq - cached).to(torch.int32))


def test_workload_length_distributions():
    s = wl.make_step(wl.BY_NAME["tiny_decode"])
    assert s.seq_len.tolist() == [5, 9, 12]
    s = wl.make_step(wl.BY_NAME["qwen3_0.6b_decode_28l"])
    assert 128 <= int(s.seq_len.min()) and int(s.seq_len.max()) <= 2048
    s = wl.make_step(wl.BY_NAME["batch256_gqa4_decode"])
    mean = float(s.seq_len.double().mean())
    assert 700 < mean < 1200 and int(s.seq_len.max()) <= 4096
    s = wl.make_step(wl.BY_NAME["longctx_gqa8_decode"])
    assert set(s.seq_len.tolist()) == {32768}
    s = wl.make_step(wl.BY_NAME["chunked_prefill_extend"])
    n = s.seq_len - s.cached_len
    assert int(s.cached_len.max()) <= 2048 and 256 <= int(n.min()) and int(n.max()) <= 1024


def test_workload_is_deterministic_and_layers_differ():
    spec = wl.BY_NAME["tiny_decode"]
    a, b = wl.make_step(spec), wl.make_step(spec)
    assert torch.equal(a.page_table, b.page_table)
    la, lb = wl.make_layer(a, 0), wl.make_layer(b, 0)
    assert torch.equal(la.q.view(torch.int16), lb.q.view(torch.int16))
    l1 = wl.make_layer(a, 1)
    assert not torch.equal(la.q.view(torch.int16), l1.q.view(torch.int16))


def test_pool_poisoned_outside_history():
    spec = wl.BY_NAME["tiny_decode"]
    step = wl.make_step(spec)
    layer = wl.make_layer(step)
    pool = wl.build_pool(step, layer.hist_slots, layer.k_hist)
    bits = wl.bits(pool)
    hist = np.zeros(spec.num_slots, bool)
    hist[layer.hist_slots.numpy()] = True
    assert (bits[~hist] == wl.NAN_BF16_BITS).all()
    assert np.isfinite(pool[torch.from_numpy(hist)].float().numpy()).all()
    # the new tokens' slots are poisoned until the store writes them
    assert (bits[step.out_loc.numpy()] == wl.NAN_BF16_BITS).all()
