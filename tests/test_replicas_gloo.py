"""The N>1 path on CPU: two gloo ranks as separate processes.

Covers what bench.py does across ranks (per-rank workloads, barrier, max of
the ranks' times, sum of their units) and the strong-scaling request shards,
with the oracle standing in for the GPU work so no GPU is needed."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

from paged_kv_attention_mg_b200.replicas import Replicas, rank_spec, shard_requests


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import oracle
    from paged_kv_attention_mg_b200 import workload as wl
    reps = Replicas(world, backend="gloo", timeout_s=60)
    try:
        # weak scaling: each rank its own replica of the workload
        spec = rank_spec(wl.BY_NAME["tiny_decode"], reps.rank)
        step = wl.make_step(spec)
        data = wl.make_layer(step)
        k = wl.build_pool(step, data.hist_slots, data.k_hist)
        v = wl.build_pool(step, data.hist_slots, data.v_hist)
        k.index_copy_(0, step.out_loc.long(), data.k_new)
        v.index_copy_(0, step.out_loc.long(), data.v_new)
        out = oracle.decode(wl.bits(data.q), wl.bits(k), wl.bits(v), step.page_table.numpy(),
                            step.table_idx.numpy(), step.seq_len.numpy(), spec.scale, threads=1)
        reps.barrier()
        fake_ms = 10.0 + 5.0 * reps.rank
        t_max = reps.max(fake_ms)
        units = reps.sum(step.batch)
        # the roofline line reports the lowest rank's own achieved rate
        rate_min = reps.min(100.0 - 30.0 * reps.rank)
        # strong scaling: one global batch, contiguous request shards
        gspec = wl.custom_spec("decode", [4, 30, 7, 99, 12], [5, 31, 8, 100, 13], 8, 2, 400, seed=5)
        gstep = wl.make_step(gspec)
        gdata = wl.make_layer(gstep)
        gk = wl.build_pool(gstep, gdata.hist_slots, gdata.k_hist)
        gv = wl.build_pool(gstep, gdata.hist_slots, gdata.v_hist)
        gk.index_copy_(0, gstep.out_loc.long(), gdata.k_new)
        gv.index_copy_(0, gstep.out_loc.long(), gdata.v_new)
        b0, b1 = shard_requests(gstep.batch, reps.rank, reps.world)
        part = oracle.decode(wl.bits(gdata.q), wl.bits(gk), wl.bits(gv), gstep.page_table.numpy(),
                             gstep.table_idx.numpy(), gstep.seq_len.numpy(), gspec.scale,
                             requests=range(b0, b1), threads=1)
        queue.put(dict(rank=reps.rank, seed=spec.seed, page_table=step.page_table.numpy(), out=out,
                       t_max=t_max, units=units, rate_min=rate_min, shard=(b0, b1), part=part))
    finally:
        reps.close()


def test_two_gloo_ranks_replicas_and_shards():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        item = queue.get(timeout=120)
        res[item["rank"]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from paged_kv_attention_mg_b200 import workload as wl
    canonical = wl.BY_NAME["tiny_decode"]
    assert res[0]["seed"] == canonical.seed and res[1]["seed"] != canonical.seed
    assert not np.array_equal(res[0]["page_table"], res[1]["page_table"])
    assert res[0]["t_max"] == res[1]["t_max"] == 15.0      # max over ranks
    assert res[0]["units"] == res[1]["units"] == 2 * canonical.batch
    assert res[0]["rate_min"] == res[1]["rate_min"] == 70.0  # min over ranks
    assert np.isfinite(res[0]["out"]).all() and np.isfinite(res[1]["out"]).all()
    # shards cover the batch once, and the union equals the single-process result
    (a0, a1), (b0, b1) = res[0]["shard"], res[1]["shard"]
    assert a0 == 0 and a1 == b0 and b1 == 5
    import oracle
    gspec = wl.custom_spec("decode", [4, 30, 7, 99, 12], [5, 31, 8, 100, 13], 8, 2, 400, seed=5)
    gstep = wl.make_step(gspec)
    gdata = wl.make_layer(gstep)
    gk = wl.build_pool(gstep, gdata.hist_slots, gdata.k_hist)
    gv = wl.build_pool(gstep, gdata.hist_slots, gdata.v_hist)
    gk.index_copy_(0, gstep.out_loc.long(), gdata.k_new)
    gv.index_copy_(0, gstep.out_loc.long(), gdata.v_new)
    full = oracle.decode(wl.bits(gdata.q), wl.bits(gk), wl.bits(gv), gstep.page_table.numpy(),
                         gstep.table_idx.numpy(), gstep.seq_len.numpy(), gspec.scale, threads=1)
    merged = np.where(np.isnan(res[0]["part"]), res[1]["part"], res[0]["part"])
    assert np.array_equal(merged, full)


@pytest.mark.parametrize("batch,world", [(5, 2), (64, 8), (3, 4), (0, 2), (256, 3)])
def test_shard_requests_partition(batch, world):
    seen = []
    for r in range(world):
        b, e = shard_requests(batch, r, world)
        assert 0 <= b <= e <= batch
        seen.extend(range(b, e))
    assert seen == list(range(batch))
    sizes = [shard_requests(batch, r, world) for r in range(world)]
    lens = [e - b for b, e in sizes]
    assert max(lens) - min(lens) <= 1


def test_single_process_needs_no_group():
    reps = Replicas(None, backend="gloo")
    assert reps.world == 1 and reps.pg is None
    assert reps.max(3.5) == 3.5 and reps.sum(2.0) == 2.0
    reps.close()


@pytest.mark.parametrize("hq,hkv,world", [(16, 8, 2), (16, 8, 8), (32, 4, 8), (16, 2, 4), (8, 8, 1), (32, 8, 4)])
def test_shard_kv_heads_partition(hq, hkv, world):
    from paged_kv_attention_mg_b200.replicas import shard_kv_heads
    g = hq // hkv
    seen = []
    for r in range(world):
        kv0, kv1, q0, q1 = shard_kv_heads(hq, hkv, r, world)
        assert 0 <= kv0 < kv1 <= hkv and 0 <= q0 < q1 <= hq
        assert all(kv0 <= h // g < kv1 for h in range(q0, q1))  # its q heads read only its KV heads
        # the local GQA mapping on the slice is the global one shifted
        gl = (q1 - q0) // (kv1 - kv0)
        assert all((h - q0) // gl == h // g - kv0 for h in range(q0, q1))
        seen.extend(range(q0, q1))
    assert sorted(seen) == list(range(hq))  # every query head on exactly one rank


def _head_rank_main(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import oracle
    import torch.distributed as dist
    from paged_kv_attention_mg_b200 import workload as wl
    from paged_kv_attention_mg_b200.replicas import shard_kv_heads, take_heads
    reps = Replicas(world, backend="gloo", timeout_s=60)
    try:
        spec = wl.custom_spec("decode", [4, 30, 7, 99, 12], [5, 31, 8, 100, 13], 8, 2, 400, seed=5)
        step = wl.make_step(spec)
        data = wl.make_layer(step)
        k = wl.build_pool(step, data.hist_slots, data.k_hist)
        v = wl.build_pool(step, data.hist_slots, data.v_hist)
        k.index_copy_(0, step.out_loc.long(), data.k_new)
        v.index_copy_(0, step.out_loc.long(), data.v_new)
        kv0, kv1, q0, q1 = shard_kv_heads(spec.num_q_heads, spec.num_kv_heads, reps.rank, reps.world)
        # this rank's slice: its query heads and a pool holding only its KV heads
        part = oracle.decode(wl.bits(take_heads(data.q, q0, q1)), wl.bits(take_heads(k, kv0, kv1)),
                             wl.bits(take_heads(v, kv0, kv1)), step.page_table.numpy(), step.table_idx.numpy(),
                             step.seq_len.numpy(), spec.scale, threads=1)
        gathered = [None] * reps.world
        dist.all_gather_object(gathered, (q0, q1, part))
        queue.put(dict(rank=reps.rank, gathered=gathered))
    finally:
        reps.close()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_kv_head_shards_reassemble_the_full_result(world):
    """Tensor-parallel attention on CPU ranks: each rank runs its KV heads (and,
    with 4 ranks over 2 KV heads, half of a replicated head's query heads) on
    its own pool slice; the gathered heads equal the single-process result bit
    for bit (every (request, head) is computed the same way either way)."""
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        item = queue.get(timeout=120)
        res[item["rank"]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    from paged_kv_attention_mg_b200 import workload as wl
    spec = wl.custom_spec("decode", [4, 30, 7, 99, 12], [5, 31, 8, 100, 13], 8, 2, 400, seed=5)
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    k = wl.build_pool(step, data.hist_slots, data.k_hist)
    v = wl.build_pool(step, data.hist_slots, data.v_hist)
    k.index_copy_(0, step.out_loc.long(), data.k_new)
    v.index_copy_(0, step.out_loc.long(), data.v_new)
    full = oracle.decode(wl.bits(data.q), wl.bits(k), wl.bits(v), step.page_table.numpy(), step.table_idx.numpy(),
                         step.seq_len.numpy(), spec.scale, threads=1)
    gathered = res[0]["gathered"]
    ranges = [(q0, q1) for (q0, q1, _) in gathered]
    assert all([(q0, q1) for (q0, q1, _) in res[r]["gathered"]] == ranges for r in res)  # same view on every rank
    out = np.concatenate([part for (_, _, part) in sorted(gathered, key=lambda t: t[0])], axis=1)
    assert np.array_equal(out, full)
