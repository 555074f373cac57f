"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

* store: bit-exact over the whole pool, unreferenced slots (NaN-poisoned)
  untouched;
* decode / extend: max |err| <= 1e-2 and mean |err| <= 1e-3 on bf16 outputs,
  on small cases spanning several tiles and ragged tails, and at the full
  workload sizes on sampled requests, in the launch configuration bench.py
  times (automatic split plan);
* invariants only the GPU path has: split-count independence, run-to-run
  determinism, device-side metadata checks that flag instead of faulting.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mg_testlib import (GpuStep, assert_matches_oracle, host_pools_after_store, oracle_decode,
                        oracle_extend)
from paged_kv_attention_mg_b200 import mg
from paged_kv_attention_mg_b200 import workload as wl

pytestmark = pytest.mark.gpu


def _custom(kind, cached, seq, hq, hkv, seed, slack=37):
    spec = wl.custom_spec(kind, cached, seq, hq, hkv, sum(seq) + slack, seed)
    step = wl.make_step(spec)
    return step, wl.make_layer(step)


# ----------------------------------------------------------------------------- store

@pytest.mark.parametrize("name", ["tiny_decode", "chunked_prefill_extend"])
def test_store_bit_exact_whole_pool(name):
    spec = wl.BY_NAME[name]
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    g = GpuStep(step, data)
    g.store()
    torch.cuda.synchronize()
    k_ref = wl.build_pool(step, data.hist_slots, data.k_hist)
    v_ref = wl.build_pool(step, data.hist_slots, data.v_hist)
    kb, vb = wl.bits(k_ref).copy(), wl.bits(v_ref).copy()
    oracle.store_kv(wl.bits(data.k_new), wl.bits(data.v_new), step.out_loc.numpy(), kb, vb)
    assert np.array_equal(wl.bits(g.k_cache.cpu()), kb)
    assert np.array_equal(wl.bits(g.v_cache.cpu()), vb)
    assert mg.read_device_error() == 0


@pytest.mark.parametrize("hkv", [1, 2, 4, 8])
def test_store_various_heads_and_ragged_counts(hkv):
    step, data = _custom("extend", [0, 7, 1], [1, 40, 300], 2 * hkv, hkv, seed=hkv)
    g = GpuStep(step, data)
    g.store()
    k_ref, v_ref = host_pools_after_store(step, data)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), v_ref.view(torch.int16))


def test_store_flags_out_of_range_slot_and_skips_it():
    step, data = _custom("extend", [0], [8], 16, 8, seed=3)
    g = GpuStep(step, data)
    bad = g.out_loc.clone()
    bad[3] = g.k_cache.shape[0] + 5
    mg.read_device_error()
    mg.store_kv(g.k_new, g.v_new, bad, g.k_cache, g.v_cache)
    assert mg.read_device_error() & mg.DEVERR_SLOT_RANGE
    # the other tokens were stored
    k = g.k_cache.cpu()
    for t in (0, 1, 2, 4, 7):
        assert torch.equal(k[int(step.out_loc[t])].view(torch.int16), data.k_new[t].view(torch.int16))


# ----------------------------------------------------------------------------- decode

DECODE_SMALL = [
    # lengths, hq, hkv
    ([5, 9, 12], 16, 8),
    ([1], 16, 8),
    ([1, 2, 3, 63, 64, 65, 129], 8, 8),
    ([300, 17, 250], 8, 2),
    ([200, 1, 77, 128], 32, 4),
    ([257, 190], 32, 2),      # group 16
    ([33, 100], 4, 4),        # group 1
    ([511, 3, 1000, 2], 12, 4),  # group 3 (not a power of two)
    ([130, 7, 400], 28, 4),   # group 7
    ([66, 300], 24, 2),       # group 12 (two row blocks, not a power of two)
]


@pytest.mark.parametrize("lengths,hq,hkv", DECODE_SMALL)
@pytest.mark.parametrize("parts", [0, 1, 7])
def test_decode_small_matches_oracle(lengths, hq, hkv, parts):
    step, data = _custom("decode", [L - 1 for L in lengths], lengths, hq, hkv, seed=len(lengths) * 31 + hq)
    g = GpuStep(step, data)
    g.store()
    out = g.decode(num_partitions=parts)
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_decode(step, data), f"decode {lengths} partitions {parts}")


def test_decode_tiny_workload():
    spec = wl.BY_NAME["tiny_decode"]
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    g = GpuStep(step, data)
    g.store()
    out = g.decode()
    assert_matches_oracle(out, oracle_decode(step, data), "tiny_decode")


def test_decode_random_sweep():
    rng = np.random.default_rng(7)
    for it in range(12):
        hkv = int(rng.choice([1, 2, 4, 8]))
        grp = int(rng.choice([1, 2, 4, 8]))
        b = int(rng.integers(1, 8))
        lengths = [int(x) for x in rng.integers(1, 301, size=b)]
        step, data = _custom("decode", [L - 1 for L in lengths], lengths, hkv * grp, hkv, seed=100 + it)
        g = GpuStep(step, data)
        g.store()
        parts = int(rng.choice([0, 1, 5, 33, 4096]))
        out = g.decode(num_partitions=parts)
        assert_matches_oracle(out, oracle_decode(step, data), f"sweep {it}: {lengths} hkv {hkv} g {grp}")


def _sample(step, k=6, seed=0):
    b = step.batch
    L = step.seq_len.numpy()
    picks = {int(np.argmax(L)), int(np.argmin(L)), 0, b - 1}
    picks |= set(int(x) for x in np.random.default_rng(seed).choice(b, size=min(k, b), replace=False))
    return sorted(picks)


@pytest.mark.parametrize("name,layer", [("qwen3_0.6b_decode_28l", 0), ("qwen3_0.6b_decode_28l", 27),
                                        ("batch256_gqa4_decode", 0), ("longctx_gqa8_decode", 0)])
def test_decode_full_size_sampled(name, layer):
    spec = wl.BY_NAME[name]
    step = wl.make_step(spec)
    data = wl.make_layer(step, layer)
    g = GpuStep(step, data)
    g.store()
    out = g.decode()  # automatic plan, as bench.py launches it
    assert mg.read_device_error() == 0
    req = _sample(step, k=4 if name.startswith("longctx") else 8)
    ref = oracle_decode(step, data, requests=req)
    assert_matches_oracle(out, ref, f"{name} layer {layer}")
    # every row is finite (no stray reads of poisoned slots anywhere)
    assert torch.isfinite(out.float()).all()


def test_decode_split_count_independence_and_determinism():
    step, data = _custom("decode", [1500, 2047, 3, 700], [1501, 2048, 4, 701], 32, 8, seed=5)
    g = GpuStep(step, data)
    g.store()
    a = g.decode(num_partitions=1).float()
    b = g.decode(num_partitions=997).float()
    c = g.decode().float()
    # different partitions change the running max each P is scaled by before
    # its bf16 rounding, so results differ by rounding noise, not by a fixed ulp
    tol = torch.maximum(a.abs(), b.abs()) * 2.0 ** -7 + 2e-3
    assert bool(((a - b).abs() <= tol).all())
    assert bool(((a - c).abs() <= tol).all())
    assert_matches_oracle(a, oracle_decode(step, data), "1 worker")
    assert_matches_oracle(b, oracle_decode(step, data), "997 workers")
    c2 = g.decode().float()
    assert torch.equal(c, c2)


@pytest.mark.parametrize("batch", [1000, 2000])
def test_decode_batch_over_one_scan_chunk(batch):
    """More requests than one prologue scan chunk holds (the second pass then
    scans every chunk that overlaps a CTA's workers instead of reusing the
    first pass), plain and fused."""
    rng = np.random.default_rng(batch)
    lengths = [int(x) for x in rng.integers(1, 200, size=batch)]
    step, data = _custom("decode", [L - 1 for L in lengths], lengths, 16, 8, seed=batch + 3)
    g = GpuStep(step, data)
    req = _sample(step, k=12, seed=batch)
    out = g.store_decode()
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_decode(step, data, requests=req), f"fused, batch {batch}")
    out2 = g.decode()  # the pools now hold the stored tokens
    assert mg.read_device_error() == 0
    assert_matches_oracle(out2, oracle_decode(step, data, requests=req), f"plain, batch {batch}")


def test_decode_with_larger_max_seq_len_hint():
    step, data = _custom("decode", [99, 5], [100, 6], 16, 8, seed=6)
    g = GpuStep(step, data)
    g.store()
    out = g.decode(max_seq_len=step.page_table.shape[1])
    assert_matches_oracle(out, oracle_decode(step, data), "hint = table width")


def test_decode_flags_bad_metadata_without_faulting():
    step, data = _custom("decode", [9, 19], [10, 20], 16, 8, seed=8)
    g = GpuStep(step, data)
    g.store()
    mg.read_device_error()
    row = int(step.table_idx[1])
    g.page_table[row, 4] = g.k_cache.shape[0] + 100  # slot outside the pool
    g.decode()
    assert mg.read_device_error() & mg.DEVERR_SLOT_RANGE
    g.page_table.copy_(step.page_table.cuda())
    g.table_idx[0] = 99  # row outside the table
    g.decode()
    assert mg.read_device_error() & mg.DEVERR_ROW_RANGE
    g.table_idx.copy_(step.table_idx.cuda())
    g.seq_len[0] = 30  # beyond the max_seq_len hint (20)
    g.decode(max_seq_len=20)
    assert mg.read_device_error() & mg.DEVERR_LENGTH


def test_decode_workspace_contents_do_not_matter():
    """mg_decode_attn reads nothing from its workspace that the same call did
    not write: a workspace full of 0xFF bytes, or one a call of a different
    plan (other batch / heads) has just used, gives the oracle's output, call
    after call."""
    lengths = [700, 3, 1500, 64, 2049]
    step, data = _custom("decode", [L - 1 for L in lengths], lengths, 32, 8, seed=123)
    g = GpuStep(step, data)
    g.store()
    ref = oracle_decode(step, data)
    parts = 37  # every long pair split over several workers
    need = mg.decode_workspace_bytes(step.batch, 32, 8, step.max_seq_len, num_partitions=parts)
    other_step, other_data = _custom("decode", [99, 4000], [100, 4001], 16, 2, seed=5)
    other = GpuStep(other_step, other_data)
    other.store()
    other_need = mg.decode_workspace_bytes(other_step.batch, 16, 2, other_step.max_seq_len, num_partitions=500)
    ws = torch.full((max(need, other_need),), 0xFF, dtype=torch.uint8, device="cuda")

    def run():
        return mg.decode_attn(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.seq_len, step.max_seq_len,
                              g.scale, num_partitions=parts, workspace=ws)

    assert_matches_oracle(run(), ref, "workspace of 0xFF bytes")
    assert_matches_oracle(run(), ref, "second call on the same workspace")
    mg.decode_attn(other.q, other.k_cache, other.v_cache, other.page_table, other.table_idx, other.seq_len,
                   other_step.max_seq_len, other.scale, num_partitions=500, workspace=ws)
    assert_matches_oracle(run(), ref, "after a call of another plan")
    assert mg.read_device_error() == 0


def test_decode_host_errors():
    step, data = _custom("decode", [299], [300], 16, 8, seed=9)
    g = GpuStep(step, data)
    assert mg.decode_workspace_bytes(1, 16, 8, 300, num_partitions=64) > 16
    with pytest.raises(mg.MgError) as e:
        mg.decode_attn(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.seq_len, 300, 0.1,
                       num_partitions=64, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 4
    qm = torch.empty(g.q.numel() + 8, dtype=torch.bfloat16, device="cuda")[1:1 + g.q.numel()].view(g.q.shape)
    with pytest.raises(mg.MgError) as e:
        mg.decode_attn(qm, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.seq_len, 300, 0.1)
    assert e.value.status == 3


# ----------------------------------------------------------------------------- fused store + decode

@pytest.mark.parametrize("lengths,hq,hkv", DECODE_SMALL)
@pytest.mark.parametrize("parts", [0, 1, 7])
def test_store_decode_fused_matches_oracle_and_stores(lengths, hq, hkv, parts):
    step, data = _custom("decode", [L - 1 for L in lengths], lengths, hq, hkv, seed=len(lengths) * 37 + hq)
    g = GpuStep(step, data)
    out = g.store_decode(num_partitions=parts)
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_decode(step, data), f"fused {lengths} partitions {parts}")
    k_ref, v_ref = host_pools_after_store(step, data)  # the pool as mg_store_kv leaves it
    assert torch.equal(g.k_cache.cpu().view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), v_ref.view(torch.int16))


@pytest.mark.parametrize("name", ["qwen3_0.6b_decode_28l", "batch256_gqa4_decode", "longctx_gqa8_decode"])
def test_store_decode_fused_full_size(name):
    spec = wl.BY_NAME[name]
    step = wl.make_step(spec)
    data = wl.make_layer(step, 3 if spec.num_layers > 3 else 0)
    g = GpuStep(step, data)
    out = g.store_decode()
    assert mg.read_device_error() == 0
    req = _sample(step, k=3 if name.startswith("longctx") else 6, seed=1)
    assert_matches_oracle(out, oracle_decode(step, data, requests=req), f"fused {name}")
    # the new tokens' slots now hold k_new / v_new
    loc = step.out_loc.long()
    assert torch.equal(g.k_cache[loc.cuda()].cpu().view(torch.int16), data.k_new.view(torch.int16))
    assert torch.equal(g.v_cache[loc.cuda()].cpu().view(torch.int16), data.v_new.view(torch.int16))


def test_store_decode_fused_equals_separate_calls():
    step, data = _custom("decode", [130, 5, 999], [131, 6, 1000], 32, 8, seed=41)
    a = GpuStep(step, data)
    a.store()
    sep = a.decode(num_partitions=9)
    b = GpuStep(step, data)
    fused = b.store_decode(num_partitions=9)
    assert torch.equal(sep, fused)  # same partition, same arithmetic order
    # pools compared as bit patterns (the NaN poison compares unequal as numbers)
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    assert torch.equal(a.v_cache.view(torch.int16), b.v_cache.view(torch.int16))


def test_store_decode_flags_out_loc_mismatch():
    step, data = _custom("decode", [9, 19], [10, 20], 16, 8, seed=42)
    g = GpuStep(step, data)
    mg.read_device_error()
    bad = g.out_loc.clone()
    bad[0] = int(step.dummy_slot)  # not the page-table entry of position L-1
    mg.store_decode_attn(g.q, g.k_new, g.v_new, bad, g.k_cache, g.v_cache, g.page_table, g.table_idx,
                         g.seq_len, 20, g.scale)
    assert mg.read_device_error() & mg.DEVERR_LENGTH


def test_store_decode_stores_the_new_token_even_if_its_table_entry_is_bad():
    """The new token's page-table entry (position L-1) outside the pool: the key
    is flagged and left out of the attention, but out_loc is valid, so the pool
    slot still receives the new K/V (as mg_store_kv would write it), never the
    zero fill of a rejected row."""
    step, data = _custom("decode", [9, 19], [10, 20], 16, 8, seed=43)
    g = GpuStep(step, data)
    mg.read_device_error()
    row = int(step.table_idx[1])
    g.page_table[row, 19] = g.k_cache.shape[0] + 7
    out = mg.store_decode_attn(g.q, g.k_new, g.v_new, g.out_loc, g.k_cache, g.v_cache, g.page_table, g.table_idx,
                               g.seq_len, 20, g.scale)
    assert mg.read_device_error() & mg.DEVERR_SLOT_RANGE
    loc = int(step.out_loc[1])
    assert torch.equal(g.k_cache[loc].cpu().view(torch.int16), data.k_new[1].view(torch.int16))
    assert torch.equal(g.v_cache[loc].cpu().view(torch.int16), data.v_new[1].view(torch.int16))
    # request 0 is untouched by request 1's bad entry
    assert_matches_oracle(out, oracle_decode(step, data, requests=[0]), "request 0 beside a bad entry")


# ----------------------------------------------------------------------------- extend

EXTEND_SMALL = [
    # cached, seq, hq, hkv
    ([0], [1], 16, 8),
    ([0], [2], 16, 8),
    ([4, 8, 11], [5, 9, 12], 16, 8),            # one new token each (decode-like)
    ([0, 3, 10], [4, 9, 140], 16, 8),
    ([0], [129], 16, 8),                        # ragged past one Q block
    ([130, 0], [300, 257], 16, 8),
    ([5, 200], [70, 333], 8, 8),                # group 1
    ([17, 0, 64], [90, 64, 300], 32, 8),        # group 4
    ([0, 100], [40, 260], 32, 4),               # group 8
    ([31], [200], 32, 2),                       # group 16
    ([10, 20], [10, 50], 16, 8),                # a request with no new tokens
    ([0, 50], [130, 300], 12, 4),               # group 3: 42 tokens fill 126 of a Q tile's 128 rows
    ([7], [260], 28, 4),                        # group 7: 18 tokens, 126 rows
    ([0, 9], [100, 200], 12, 1),                # group 12: 10 tokens, 120 rows
]


@pytest.mark.parametrize("cached,seq,hq,hkv", EXTEND_SMALL)
def test_extend_small_matches_oracle(cached, seq, hq, hkv):
    step, data = _custom("extend", cached, seq, hq, hkv, seed=sum(seq) + hq)
    g = GpuStep(step, data)
    g.store()
    out = g.extend()
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_extend(step, data), f"extend {cached}->{seq} hq{hq} hkv{hkv}")


def test_extend_random_sweep():
    rng = np.random.default_rng(11)
    for it in range(8):
        hkv = int(rng.choice([2, 4, 8]))
        grp = int(rng.choice([1, 2, 4]))
        b = int(rng.integers(1, 5))
        cached = [int(x) for x in rng.integers(0, 400, size=b)]
        seq = [c + int(rng.integers(1, 300)) for c in cached]
        step, data = _custom("extend", cached, seq, hkv * grp, hkv, seed=200 + it)
        g = GpuStep(step, data)
        g.store()
        out = g.extend()
        assert_matches_oracle(out, oracle_extend(step, data), f"extend sweep {it}")


def test_extend_full_size_sampled():
    spec = wl.BY_NAME["chunked_prefill_extend"]
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    g = GpuStep(step, data)
    g.store()
    out = g.extend()
    assert mg.read_device_error() == 0
    n = (step.seq_len - step.cached_len).numpy()
    req = sorted({int(np.argmax(step.seq_len.numpy())), int(np.argmin(n)), 3})
    assert_matches_oracle(out, oracle_extend(step, data, requests=req), "chunked_prefill_extend")
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("cached,seq,hq,hkv", [
    ([30000, 5], [30070, 40], 16, 8),     # a chunk after a 30k-token history: 235 KV tiles an item
    ([0, 100], [2048, 101], 32, 4),       # a 2048-token fresh prompt (many q blocks) beside one token
    ([16000], [16070], 64, 8),            # group 8: 16 tokens a Q tile, ragged last q block
])
def test_extend_long_items(cached, seq, hq, hkv):
    """Items far longer than the chunked-prefill workload's: long KV loops per
    item and prompts of many q blocks, checked against the oracle."""
    step, data = _custom("extend", cached, seq, hq, hkv, seed=sum(seq) % 1000 + 5)
    g = GpuStep(step, data)
    g.store()
    out = g.extend()
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_extend(step, data), f"extend long {cached}->{seq} hq {hq} hkv {hkv}")


def test_extend_single_token_matches_decode_kernel():
    lengths = [5, 64, 129, 300]
    step, data = _custom("decode", [L - 1 for L in lengths], lengths, 16, 8, seed=12)
    g = GpuStep(step, data)
    g.store()
    dec = g.decode().float()
    ext = g.extend().float()
    assert bool(((dec - ext).abs() <= dec.abs() * 2.0 ** -7 + 2e-3).all())


def test_extend_deterministic():
    step, data = _custom("extend", [100, 0], [400, 200], 16, 8, seed=13)
    g = GpuStep(step, data)
    g.store()
    a = g.extend()
    b = g.extend()
    assert torch.equal(a, b)


@pytest.mark.parametrize("batch", [250, 300])
def test_extend_work_list_sorted_or_walked(batch):
    """The kernel sorts the (request, q block) groups that hold tokens when
    there are at most 256 of them, and walks the plain enumeration otherwise:
    250 and 300 short prompts (one group each) take the two paths, with
    requests that have nothing new in between."""
    rng = np.random.default_rng(batch)
    cached = [int(x) for x in rng.integers(0, 200, size=batch)]
    seq = [c + int(rng.integers(1, 40)) for c in cached]
    for r in range(0, batch, 17):
        seq[r] = cached[r]  # no new token: no group
    step, data = _custom("extend", cached, seq, 16, 8, seed=900 + batch)
    g = GpuStep(step, data)
    g.store()
    out = g.extend()
    assert mg.read_device_error() == 0
    req = sorted(set(range(0, batch, 23)) | {1, batch - 1})
    assert_matches_oracle(out, oracle_extend(step, data, requests=req), f"extend, {batch} short prompts")


# --------------------------------------------------------------------------- tensor-parallel head shards

@pytest.mark.parametrize("world", [2, 16])
def test_kv_head_shards_through_the_unchanged_kernels(world):
    """A tensor-parallel rank's slice -- its query heads and a pool holding only
    its KV heads (world 16 over 8 KV heads: each head on two ranks, half its
    query heads each) -- through decode, fused store+decode and extend gives the
    oracle's rows for those heads."""
    from paged_kv_attention_mg_b200.replicas import shard_kv_heads, take_heads
    hq, hkv = 32, 8
    lengths = [700, 3, 1500, 64, 2049]
    dstep, ddata = _custom("decode", [L - 1 for L in lengths], lengths, hq, hkv, seed=321)
    dref = oracle_decode(dstep, ddata)
    estep, edata = _custom("extend", [0, 130, 900], [150, 400, 1000], hq, hkv, seed=322)
    eref = oracle_extend(estep, edata)
    for r in range(world):
        kv0, kv1, q0, q1 = shard_kv_heads(hq, hkv, r, world)
        # decode and fused store+decode on the rank's own pool slice (new token not yet stored)
        d = GpuStep(dstep, ddata)
        kc, vc = take_heads(d.k_cache, kv0, kv1), take_heads(d.v_cache, kv0, kv1)
        q = take_heads(d.q, q0, q1)
        out = mg.store_decode_attn(q, take_heads(d.k_new, kv0, kv1), take_heads(d.v_new, kv0, kv1), d.out_loc,
                                   kc, vc, d.page_table, d.table_idx, d.seq_len, dstep.max_seq_len, d.scale)
        assert_matches_oracle(out, dref[:, q0:q1], f"rank {r}/{world} fused store+decode heads {q0}..{q1}")
        out = mg.decode_attn(q, kc, vc, d.page_table, d.table_idx, d.seq_len, dstep.max_seq_len, d.scale)
        assert_matches_oracle(out, dref[:, q0:q1], f"rank {r}/{world} decode heads {q0}..{q1}")
        # extend
        e = GpuStep(estep, edata)
        e.store()
        out = mg.extend_attn(take_heads(e.q, q0, q1), take_heads(e.k_cache, kv0, kv1), take_heads(e.v_cache, kv0, kv1),
                             e.page_table, e.table_idx, e.cached_len, e.seq_len, e.q_offset, estep.max_q_len,
                             estep.max_seq_len, e.scale)
        assert_matches_oracle(out, eref[:, q0:q1], f"rank {r}/{world} extend heads {q0}..{q1}")
    assert mg.read_device_error() == 0


def test_extend_serves_a_mixed_batch():
    """One mg_extend_attn launch over a batch as a chunked-prefill scheduler forms
    it: decode requests (one new token after a long history), chunks of a
    prompt, a fresh prompt and a request with nothing new this step."""
    cached = [1999, 0, 512, 3000, 77, 40]
    seq = [2000, 700, 1024, 3001, 78, 40]  # n = 1, 700, 512, 1, 1, 0
    step, data = _custom("extend", cached, seq, 16, 8, seed=404)
    g = GpuStep(step, data)
    g.store()
    out = g.extend()
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_extend(step, data), "mixed decode / prefill batch")


def test_extend_serves_the_mixed_workload():
    """The mixed_prefill_decode workload in one mg_extend_attn launch: 200
    one-token decode requests and 4 prompt chunks, each decode request an item
    of its own in the persistent kernel's work list (its padding rows skipped).
    Sampled rows against the oracle; every decode row also against the decode
    kernel on the same pool."""
    spec = wl.BY_NAME["mixed_prefill_decode"]
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    g = GpuStep(step, data)
    g.store()
    out = g.extend()
    assert mg.read_device_error() == 0
    assert torch.isfinite(out.float()).all()
    req = [0, 1, 2, 3] + list(range(4, 204, 13))
    assert_matches_oracle(out, oracle_extend(step, data, requests=req), "mixed_prefill_decode")
    # decode requests (rows q_offset[r] of out) equal the decode kernel's rows
    dec_rows = step.q_offset[4:204].long()
    dq = g.q[dec_rows.cuda()].contiguous()
    ti, sl = g.table_idx[4:].contiguous(), g.seq_len[4:].contiguous()
    dec = mg.decode_attn(dq, g.k_cache, g.v_cache, g.page_table, ti, sl, step.max_seq_len, g.scale).float()
    ext = out[dec_rows.cuda()].float()
    assert bool(((dec - ext).abs() <= dec.abs() * 2.0 ** -7 + 2e-3).all())


MIXED_SMALL = [
    # cached, seq: one-token requests beside chunks, a request with no new tokens, a fresh prompt
    ([1999, 0, 512, 3000, 77, 40], [2000, 700, 1024, 3001, 78, 40]),
    ([5, 0, 130], [6, 1, 131]),                 # every request one token (decode only)
    ([0, 300], [260, 500]),                     # no one-token request (extend only)
]


@pytest.mark.parametrize("cached,seq", MIXED_SMALL)
@pytest.mark.parametrize("parts,ectas", [(0, 0), (7, 0), (0, 20), (7, 1), (0, 400)])
def test_mixed_attn_matches_oracle(cached, seq, parts, ectas):
    """Both halves one after the other (extend_ctas 0) and side by side on
    split SMs (a few, one, more than the GPU has)."""
    step, data = _custom("extend", cached, seq, 16, 8, seed=sum(seq) + parts)
    g = GpuStep(step, data)
    g.store()
    out = mg.mixed_attn(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.cached_len, g.seq_len, g.q_offset,
                        max(step.max_q_len, 1), step.max_seq_len, g.scale, num_partitions=parts, extend_ctas=ectas)
    torch.cuda.synchronize()
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_extend(step, data), f"mixed {cached}->{seq} partitions {parts} ectas {ectas}")


def test_mixed_attn_on_the_mixed_workload():
    """The mixed workload through mg_mixed_attn (decode kernel for its 200
    one-token requests, extend kernel for its 4 chunks) matches the oracle on
    sampled requests and the single extend launch row for row."""
    spec = wl.BY_NAME["mixed_prefill_decode"]
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    g = GpuStep(step, data)
    g.store()
    out = mg.mixed_attn(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.cached_len, g.seq_len, g.q_offset,
                        step.max_q_len, step.max_seq_len, g.scale)
    assert mg.read_device_error() == 0
    req = [0, 1, 2, 3] + list(range(4, 204, 11))
    assert_matches_oracle(out, oracle_extend(step, data, requests=req), "mixed_attn, mixed_prefill_decode")
    ext = g.extend().float()
    assert bool(((out.float() - ext).abs() <= ext.abs() * 2.0 ** -7 + 2e-3).all())
    # the same call with the two kernels side by side on split SMs, at the split
    # the bench times: the same rows as the sequential call, bit for bit (each
    # row is computed by the same kernel either way)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ectas = mg.mixed_extend_ctas(step.cached_len.tolist(), step.seq_len.tolist(), spec.num_q_heads,
                                 spec.num_kv_heads, sms)
    assert 0 < ectas < sms
    split = mg.mixed_attn(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.cached_len, g.seq_len,
                          g.q_offset, step.max_q_len, step.max_seq_len, g.scale, extend_ctas=ectas)
    torch.cuda.synchronize()
    assert mg.read_device_error() == 0
    ext_rows = torch.zeros(out.shape[0], dtype=torch.bool)
    for r in range(4):
        ext_rows[int(step.q_offset[r]):int(step.q_offset[r + 1])] = True
    assert torch.equal(split[ext_rows.cuda()], out[ext_rows.cuda()])
    assert_matches_oracle(split, oracle_extend(step, data, requests=req), "mixed_attn split, mixed_prefill_decode")


def test_mixed_attn_split_under_graph_capture():
    """The split call (extend kernel on a side stream forked and joined with
    events) captured in a CUDA graph and replayed gives the eager call's
    output bit for bit, on fresh inputs copied into the captured buffers."""
    spec = wl.BY_NAME["mixed_prefill_decode"]
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    g = GpuStep(step, data)
    g.store()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ectas = mg.mixed_extend_ctas(step.cached_len.tolist(), step.seq_len.tolist(), spec.num_q_heads,
                                 spec.num_kv_heads, sms)
    ws = torch.empty(mg.mixed_workspace_bytes(step.batch, spec.num_q_heads, spec.num_kv_heads, step.max_seq_len),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(g.q)

    def call():
        mg.mixed_attn(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.cached_len, g.seq_len, g.q_offset,
                      step.max_q_len, step.max_seq_len, g.scale, extend_ctas=ectas, out=out, workspace=ws)
    call()  # eager, also creates the library's side stream before the capture
    torch.cuda.synchronize()
    q0 = g.q.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    q1 = torch.randn(g.q.shape, generator=torch.Generator().manual_seed(77)).to(torch.bfloat16).cuda()
    for q in (q0, q1):
        g.q.copy_(q)
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        replayed = out.clone()
        out.zero_()
        call()
        torch.cuda.synchronize()
        assert mg.read_device_error() == 0
        assert torch.equal(replayed, out)
    del graph


# --------------------------------------------------------------------------- shared prefix

def test_decode_and_extend_over_a_shared_prefix():
    """Requests whose page-table rows begin with the same slots (a prefix cache
    hit: one copy of the shared tokens in the pool) read those slots through
    every row; decode, fused store+decode and extend match the oracle on the
    same tables.  (The kernels read the shared keys once per request; reading
    them once per group is not built.)"""
    prefix = 1500
    lengths = [prefix + 40, prefix + 1, prefix + 700, prefix + 129, 300]
    step, data = _custom("decode", [L - 1 for L in lengths], lengths, 32, 8, seed=777)
    pt, ti = step.page_table, step.table_idx.long()
    for r in (1, 2, 3):  # requests 1-3 share request 0's first `prefix` slots
        pt[ti[r], :prefix] = pt[ti[0], :prefix]
    ref = oracle_decode(step, data)
    g = GpuStep(step, data)
    assert_matches_oracle(g.store_decode(), ref, "fused store+decode, shared prefix")
    assert_matches_oracle(g.decode(num_partitions=61), ref, "decode, shared prefix, 61 workers")
    ecached = [prefix, prefix + 64, prefix, 0]
    eseq = [prefix + 200, prefix + 100, prefix + 1, 180]
    estep, edata = _custom("extend", ecached, eseq, 16, 8, seed=778)
    ept, eti = estep.page_table, estep.table_idx.long()
    for r in (1, 2):
        ept[eti[r], :prefix] = ept[eti[0], :prefix]
    e = GpuStep(estep, edata)
    e.store()
    assert_matches_oracle(e.extend(), oracle_extend(estep, edata), "extend, shared prefix")
    assert mg.read_device_error() == 0
