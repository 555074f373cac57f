"""GPU: decode over shared prefixes read once per group (mg_decode_attn_shared_prefix,
and mg_store_decode_attn_shared_prefix with the KV store fused in).

Requests that share the beginning of their history, as a radix prefix cache
hands it out ("Mini-SGLang" tag page, KV Cache post), have page-table rows that
begin with the same slots.  The shared-prefix decode reads those K/V rows once
per group and KV head for every member's q heads, then merges that partial
result with each request's own keys.  Its output must be the plain decode's:
held to the oracle (which knows nothing of groups and reads every row in
full), on small cases, forced worker counts, malformed groups (served as plain
requests and flagged) and the full-size shared-prefix workload.
"""
import numpy as np
import pytest
import torch

from mg_testlib import GpuStep, assert_matches_oracle, host_pools_after_store, oracle_decode
from paged_kv_attention_mg_b200 import mg
from paged_kv_attention_mg_b200 import workload as wl

pytestmark = pytest.mark.gpu


def _grouped_case(lengths, groups, hq, hkv, seed):
    """groups: list of (first, count, P); requests outside every group are
    singletons with no shared prefix.  Rows of a group share the first
    member's first P slots; the pool is drawn after the rows are shared."""
    spec = wl.custom_spec("decode", [L - 1 for L in lengths], lengths, hq, hkv, sum(lengths) + 41, seed)
    step = wl.make_step(spec)
    firsts, plen, covered = [], [], set()
    r = 0
    groups = sorted(groups)
    gi = 0
    while r < step.batch:
        if gi < len(groups) and groups[gi][0] == r:
            g0, cnt, P = groups[gi]
            lead = int(step.table_idx[g0])
            for m in range(g0 + 1, g0 + cnt):
                step.page_table[int(step.table_idx[m]), :P] = step.page_table[lead, :P]
            firsts.append(g0)
            plen.append(P)
            r = g0 + cnt
            gi += 1
        else:
            firsts.append(r)
            plen.append(0)
            r += 1
    firsts.append(step.batch)
    step.group_first = torch.tensor(firsts, dtype=torch.int32)
    step.prefix_len = torch.tensor(plen, dtype=torch.int32)
    return step, wl.make_layer(step)


def _run(g: GpuStep, step, parts=0, group_first=None, prefix_len=None):
    gf = (step.group_first if group_first is None else group_first).cuda()
    pl = (step.prefix_len if prefix_len is None else prefix_len).cuda()
    return mg.decode_attn_shared_prefix(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.seq_len, gf, pl,
                                        step.max_seq_len, g.scale, num_partitions=parts)


# three groups of four requests sharing 1500-token prefixes, two plain requests
LENGTHS = [1540, 1501, 2200, 1629, 1900, 1777, 1502, 3000, 1501, 1600, 2048, 1530, 300, 2100]
GROUPS = [(0, 4, 1500), (4, 4, 1500), (8, 4, 1500)]


@pytest.mark.parametrize("parts", [0, 1, 37, 997])
def test_shared_prefix_decode_matches_the_oracle(parts):
    step, data = _grouped_case(LENGTHS, GROUPS, 32, 8, seed=611)  # group 4: four members fill 16 rows
    g = GpuStep(step, data)
    g.store()
    ref = oracle_decode(step, data)
    out = _run(g, step, parts)
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, ref, f"shared prefix, {parts} workers")
    plain = g.decode(num_partitions=parts).float()
    assert bool(((out.float() - plain).abs() <= plain.abs() * 2.0 ** -7 + 2e-3).all())


@pytest.mark.parametrize("hq,hkv,members", [(16, 8, 8), (8, 8, 16), (32, 4, 2), (24, 2, 1)])
def test_shared_prefix_group_sizes(hq, hkv, members):
    """Groups as large as 16 q rows allow (16 / group members), and a group of one."""
    n = members + 2
    rng = np.random.default_rng(hq * 7 + members)
    lengths = [int(x) for x in 700 + rng.integers(1, 400, size=n)]
    step, data = _grouped_case(lengths, [(1, members, 650)], hq, hkv, seed=612 + members)
    g = GpuStep(step, data)
    g.store()
    out = _run(g, step, parts=0)
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_decode(step, data), f"Hq {hq} Hkv {hkv}, {members} members")


def test_malformed_groups_are_flagged_and_served_as_plain_requests():
    step, data = _grouped_case(LENGTHS, GROUPS, 32, 8, seed=613)
    g = GpuStep(step, data)
    g.store()
    ref = oracle_decode(step, data)
    mg.read_device_error()
    # five members for group 4 (16 / 4 = 4 allowed): the first two groups merged
    gf = torch.tensor([0, 5, 8, 12, 13, 14], dtype=torch.int32)
    pl = torch.tensor([1500, 1500, 1500, 0, 0], dtype=torch.int32)
    out = _run(g, step, group_first=gf, prefix_len=pl)
    assert mg.read_device_error() & mg.DEVERR_LENGTH
    assert_matches_oracle(out, ref, "a group with too many members")
    # a prefix as long as a member's whole history (1501 = that request's seq_len)
    pl = step.prefix_len.clone()
    pl[2] = 1501
    out = _run(g, step, prefix_len=pl)
    assert mg.read_device_error() & mg.DEVERR_LENGTH
    assert_matches_oracle(out, ref, "a prefix that leaves a member no token of its own")
    # a shorter prefix than the rows share is still exact (the rest is each request's own)
    pl = step.prefix_len.clone()
    pl[0] = 700
    out = _run(g, step, prefix_len=pl)
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, ref, "a prefix shorter than the shared slots")


def test_shared_prefix_workload_full_size():
    spec = wl.BY_NAME["shared_prefix_decode"]
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    g = GpuStep(step, data)
    g.store()
    out = _run(g, step)
    assert mg.read_device_error() == 0
    req = sorted({0, 1, 7, 8, 30, 63, int(np.argmax(step.seq_len.numpy()))})
    assert_matches_oracle(out, oracle_decode(step, data, requests=req), "shared_prefix_decode")
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("groups", [100, 150])
def test_many_groups_cached_and_not(groups):
    """Many small groups: up to 128 have their ranges and prefixes checked once
    into shared memory, more are looked up in global memory; both give the
    oracle's result (sampled requests)."""
    rng = np.random.default_rng(groups)
    lengths = [int(x) for x in 200 + rng.integers(1, 300, size=2 * groups)]
    grp = [(2 * i, 2, 150 + (i % 40)) for i in range(groups)]
    step, data = _grouped_case(lengths, grp, 16, 8, seed=620 + groups)
    g = GpuStep(step, data)
    g.store()
    out = _run(g, step)
    assert mg.read_device_error() == 0
    req = sorted({0, 1, 2, 77, 128, 129, 2 * groups - 1} & set(range(step.batch)))
    assert_matches_oracle(out, oracle_decode(step, data, requests=req), f"{groups} groups")


def _run_fused(g: GpuStep, step, parts=0, group_first=None, prefix_len=None):
    gf = (step.group_first if group_first is None else group_first).cuda()
    pl = (step.prefix_len if prefix_len is None else prefix_len).cuda()
    return mg.store_decode_attn_shared_prefix(g.q, g.k_new, g.v_new, g.out_loc, g.k_cache, g.v_cache, g.page_table,
                                              g.table_idx, g.seq_len, gf, pl, step.max_seq_len, g.scale,
                                              num_partitions=parts)


@pytest.mark.parametrize("parts", [0, 1, 37])
def test_fused_store_shared_prefix_matches_oracle_and_stores(parts):
    """The KV store fused into the shared-prefix decode: the result is the
    oracle's over the pool after the store, and the pool afterwards is, bit
    for bit, the one mg_store_kv leaves (the new tokens lie after every
    group's prefix, in each request's own keys)."""
    step, data = _grouped_case(LENGTHS, GROUPS, 32, 8, seed=615)
    g = GpuStep(step, data)  # pools before the store
    out = _run_fused(g, step, parts)
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_decode(step, data), f"fused shared prefix, {parts} workers")
    k_ref, v_ref = host_pools_after_store(step, data)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), v_ref.view(torch.int16))


def test_fused_store_shared_prefix_with_malformed_groups():
    """A malformed group's members are served as plain requests; their new
    tokens are stored all the same."""
    step, data = _grouped_case(LENGTHS, GROUPS, 32, 8, seed=616)
    g = GpuStep(step, data)
    mg.read_device_error()
    gf = torch.tensor([0, 5, 8, 12, 13, 14], dtype=torch.int32)  # five members of group 4: too many
    pl = torch.tensor([1500, 1500, 1500, 0, 0], dtype=torch.int32)
    out = _run_fused(g, step, group_first=gf, prefix_len=pl)
    assert mg.read_device_error() & mg.DEVERR_LENGTH
    assert_matches_oracle(out, oracle_decode(step, data), "fused, a group with too many members")
    k_ref, v_ref = host_pools_after_store(step, data)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), v_ref.view(torch.int16))


def test_fused_store_shared_prefix_workload_full_size():
    spec = wl.BY_NAME["shared_prefix_decode"]
    step = wl.make_step(spec)
    data = wl.make_layer(step)
    g = GpuStep(step, data)
    out = _run_fused(g, step)
    assert mg.read_device_error() == 0
    req = sorted({0, 1, 7, 8, 30, 63, int(np.argmax(step.seq_len.numpy()))})
    assert_matches_oracle(out, oracle_decode(step, data, requests=req), "fused shared_prefix_decode")
    loc = step.out_loc.long()
    assert torch.equal(g.k_cache[loc.cuda()].cpu().view(torch.int16), data.k_new.view(torch.int16))
    assert torch.equal(g.v_cache[loc.cuda()].cpu().view(torch.int16), data.v_new.view(torch.int16))


def test_shared_prefix_host_errors():
    step, data = _grouped_case(LENGTHS, GROUPS, 32, 8, seed=614)
    g = GpuStep(step, data)
    need = mg.decode_shared_prefix_workspace_bytes(step.batch, 5, 32, 8, step.max_seq_len)
    assert need > mg.decode_workspace_bytes(step.batch, 32, 8, step.max_seq_len)
    with pytest.raises(mg.MgError) as e:
        mg.decode_attn_shared_prefix(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.seq_len,
                                     step.group_first.cuda(), step.prefix_len.cuda(), step.max_seq_len, g.scale,
                                     workspace=torch.empty(need - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 4
