"""The C ABI library, without a GPU: it builds, loads, exports exactly what
include/mg.h declares, and rejects bad arguments on the host before any CUDA
work (these calls return before touching the device)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from paged_kv_attention_mg_b200 import build, mg

HEADER = os.path.join(build.INCLUDE, "mg.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mg_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return mg.load()


def test_header_and_binding_agree():
    assert declared_functions() == sorted(mg.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", mg.LIBRARY], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (mg_\w+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported
    for name in declared_functions():
        assert hasattr(lib, name)


def test_build_targets_sm100a_only():
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags and "-lineinfo" in flags
    assert flags.count("-gencode") == 1


def test_status_strings(lib):
    for code, name in mg.STATUS.items():
        assert lib.mg_status_string(code).decode() == name
    assert lib.mg_abi_version() == 2


def test_store_zero_tokens_is_noop(lib):
    assert lib.mg_store_kv(None, None, None, 0, None, None, 10, 8, 128, None) == 0


@pytest.mark.parametrize("args,expect", [
    (dict(num_tokens=-1), 1),
    (dict(num_slots=0), 1),
    (dict(num_kv_heads=0), 1),
    (dict(k=None), 1),
    (dict(num_kv_heads=1, head_dim=4), 2),   # 8-byte rows are not 16-byte vectors
    (dict(k=8), 3),                          # misaligned
])
def test_store_host_validation(lib, args, expect):
    base = dict(k=4096, v=4096, out_loc=4096, num_tokens=3, k_cache=4096, v_cache=4096, num_slots=10,
                num_kv_heads=8, head_dim=128)
    base.update(args)
    st = lib.mg_store_kv(base["k"], base["v"], base["out_loc"], base["num_tokens"], base["k_cache"],
                         base["v_cache"], base["num_slots"], base["num_kv_heads"], base["head_dim"], None)
    assert st == expect


@pytest.mark.parametrize("hq,hkv,d,expect", [(16, 8, 64, 2), (12, 8, 128, 2), (64, 2, 128, 2),
                                             (0, 8, 128, 1)])
def test_decode_rejects_shapes(lib, hq, hkv, d, expect):
    st = lib.mg_decode_attn(4096, 4096, 4096, 100, 4096, 5, 32, 4096, 4096, 4, 32, hq, hkv, d, 0.1, 0,
                            4096, None, 0, None)
    assert st == expect


def test_decode_rejects_bad_hints(lib):
    # max_seq_len above the page-table width
    assert lib.mg_decode_attn(4096, 4096, 4096, 100, 4096, 5, 32, 4096, 4096, 4, 33, 16, 8, 128, 0.1, 0,
                              4096, None, 0, None) == 1
    # negative partition count
    assert lib.mg_decode_attn(4096, 4096, 4096, 100, 4096, 5, 4096, 4096, 4096, 4, 4096, 16, 8, 128, 0.1,
                              -3, 4096, None, 0, None) == 1
    # batch beyond the in-kernel scan capacity
    assert lib.mg_decode_attn(4096, 4096, 4096, 100, 4096, 5, 4096, 4096, 4096, 131073, 4096, 16, 8, 128,
                              0.1, 8, 4096, 4096, 1 << 40, None) == 2


def test_decode_plan_with_forced_partitions_needs_no_device(lib):
    workers, slots = ctypes.c_int32(), ctypes.c_int64()
    assert lib.mg_decode_plan(8, 4, 32768, 1000, ctypes.byref(workers), ctypes.byref(slots)) == 0
    assert workers.value == 1000 and slots.value == 8 * 4 + 1000
    # prefix (B+1 int64, 256-aligned) + lse (slots x g fp32, 256-aligned) + partial O (slots x g x 128 fp32)
    g = 32 // 4
    a256 = lambda x: (x + 255) // 256 * 256
    want = a256(9 * 8) + a256(1032 * g * 4) + 1032 * g * 128 * 4
    assert lib.mg_decode_workspace_bytes(8, 32, 4, 128, 32768, 1000) == want
    assert lib.mg_decode_workspace_bytes(8, 12, 8, 128, 32768, 1000) == 0  # unsupported shape


def test_shared_prefix_workspace_and_host_validation(lib):
    # 5 requests + 2 groups = 7 virtual requests; rows per slot = 16 (a group's q rows)
    slots = 7 * 4 + 1000
    a256 = lambda x: (x + 255) // 256 * 256
    want = a256(8 * 8) + a256(slots * 16 * 4) + slots * 16 * 128 * 4
    assert lib.mg_decode_shared_prefix_workspace_bytes(5, 2, 32, 4, 128, 4096, 1000) == want
    assert lib.mg_decode_shared_prefix_workspace_bytes(5, 0, 32, 4, 128, 4096, 1000) == 0   # no groups
    assert lib.mg_decode_shared_prefix_workspace_bytes(5, 2, 12, 8, 128, 4096, 1000) == 0   # unsupported shape
    args = [4096, 4096, 4096, 100, 4096, 6, 32, 4096, 4096, 5, 32]
    tail = [16, 8, 128, 0.1, 1000, 4096, 4096, 1 << 30, None]
    assert lib.mg_decode_attn_shared_prefix(*args, None, 4096, 2, *tail) == 1      # no group_first
    assert lib.mg_decode_attn_shared_prefix(*args, 4096, 4096, 0, *tail) == 1      # no groups
    small = tail[:-2] + [16, None]
    assert lib.mg_decode_attn_shared_prefix(*args, 4096, 4096, 2, *small) == 4     # workspace too small


def test_mixed_extend_ctas_split_estimate():
    """mixed_extend_ctas (host logic, no device): no split without both kinds of
    request, a split inside [1, sms - 1] otherwise, and more SMs for the extend
    kernel as the prompt chunks grow against the same decode rows."""
    dec_c, dec_s = [1000] * 50, [1001] * 50
    assert mg.mixed_extend_ctas(dec_c, dec_s, 16, 8, 148) == 0                  # decode only
    assert mg.mixed_extend_ctas([0, 100], [512, 900], 16, 8, 148) == 0          # chunks only
    assert mg.mixed_extend_ctas([5], [5], 16, 8, 148) == 0                      # nothing new
    prev = 0
    for n in (64, 256, 1024, 4096, 16384):
        e = mg.mixed_extend_ctas([0] + dec_c, [n] + dec_s, 16, 8, 148)
        assert 1 <= e <= 147 and e >= prev
        prev = e
    assert prev > 74  # a chunk far heavier than the decode rows gets most of the SMs
    assert mg.mixed_extend_ctas([0] + dec_c, [256] + dec_s, 16, 8, 2) == 1     # two SMs: one each


def test_mixed_attn_host_validation(lib):
    assert lib.mg_mixed_workspace_bytes(8, 32, 4, 128, 32768, 1000) == lib.mg_decode_workspace_bytes(8, 32, 4, 128,
                                                                                                       32768, 1000)
    args = [4096, 4096, 4096, 100, 4096, 5, 32, 4096, 4096, 4096, 4096, 4, 10, 4, 32, 16, 8]
    assert lib.mg_mixed_attn(*args, 64, 0.1, 0, 0, 4096, 4096, 1 << 30, None) == 2            # head_dim 64
    assert lib.mg_mixed_attn(*args, 128, -1.0, 0, 0, 4096, 4096, 1 << 30, None) == 1          # scale
    assert lib.mg_mixed_attn(*args, 128, 0.1, 0, -1, 4096, 4096, 1 << 30, None) == 1          # extend_ctas < 0
    no_tokens = [4096, 4096, 4096, 100, 4096, 5, 32, 4096, 4096, 4096, 4096, 4, 0, 0, 32, 16, 8]
    assert lib.mg_mixed_attn(*no_tokens, 128, 0.1, 0, 0, 4096, None, 0, None) == 0            # nothing to do
    assert lib.mg_mixed_attn(*args, 128, 0.1, 1000, 0, 4096, 4096, 16, None) == 4             # workspace too small


def test_extend_rejects_shapes_and_empty_is_noop(lib):
    assert lib.mg_extend_attn(4096, 4096, 4096, 100, 4096, 5, 32, 4096, 4096, 4096, 4096, 4, 10, 4, 32,
                              16, 8, 64, 0.1, 4096, None) == 2
    # no new tokens at all: nothing to launch
    assert lib.mg_extend_attn(4096, 4096, 4096, 100, 4096, 5, 32, 4096, 4096, 4096, 4096, 4, 0, 0, 32,
                              16, 8, 128, 0.1, 4096, None) == 0


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(mg, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        mg.load(str(tmp_path / "missing.so"))


@pytest.mark.parametrize("scale", [0.0, -0.1, float("nan"), float("inf")])
def test_attention_rejects_a_scale_that_is_not_finite_and_positive(lib, scale):
    assert lib.mg_decode_attn(4096, 4096, 4096, 100, 4096, 5, 32, 4096, 4096, 4, 32, 16, 8, 128, scale, 0,
                              4096, None, 0, None) == 1
    assert lib.mg_extend_attn(4096, 4096, 4096, 100, 4096, 5, 32, 4096, 4096, 4096, 4096, 4, 0, 0, 32,
                              16, 8, 128, scale, 4096, None) == 1


def test_decode_partial_slots_cover_every_segment(lib):
    """The plan's slot count holds every split segment: units (16 keys of one
    (request, kv head) pair, request-major) are cut into equal contiguous worker
    shares [floor(wT/W), floor((w+1)T/W)); a segment is a (pair, worker) overlap
    and writes its partial to slot pair + worker, which must be unique and below
    the slot count the library reports."""
    import numpy as np
    rng = np.random.default_rng(5)
    for _ in range(40):
        batch = int(rng.integers(1, 9))
        hkv = int(rng.choice([1, 2, 4, 8]))
        lengths = [int(x) for x in rng.integers(1, 700, size=batch)]
        workers = int(rng.integers(1, 300))
        w_out, s_out = ctypes.c_int32(), ctypes.c_int64()
        assert lib.mg_decode_plan(batch, hkv, max(lengths), workers, ctypes.byref(w_out), ctypes.byref(s_out)) == 0
        W, slots = w_out.value, s_out.value
        assert W == workers
        tiles = [(L + 15) // 16 for L in lengths]
        pair_end = np.cumsum([t for t in tiles for _ in range(hkv)])   # end unit of every pair
        T = int(pair_end[-1])
        used = set()
        for w in range(W):
            u0, u1 = w * T // W, (w + 1) * T // W
            u = u0
            while u < u1:
                pair = int(np.searchsorted(pair_end, u, side="right"))
                end = min(u1, int(pair_end[pair]))
                slot = pair + w
                assert slot not in used and 0 <= slot < slots
                used.add(slot)
                u = end


def test_binding_checks_the_sizes_the_library_takes_on_trust():
    """The C ABI trusts the pool, output and metadata sizes it is given, so the
    binding compares tensor shapes before any pointer is passed (host tensors
    suffice: the shape checks come first)."""
    bf, i32 = torch.bfloat16, torch.int32
    b, hq, hkv, d, slots = 3, 8, 4, 128, 50
    q = torch.zeros(b, hq, d, dtype=bf)
    k = torch.zeros(slots, hkv, d, dtype=bf)
    pt = torch.zeros(b + 1, 32, dtype=i32)
    idx = torch.arange(b, dtype=i32)
    seq = torch.ones(b, dtype=i32)
    cases = [
        (lambda: mg.decode_attn(q, k, k[:-1], pt, idx, seq, 16, 0.1), "v_cache"),
        (lambda: mg.decode_attn(q, k, k, pt, idx, seq[:-1], 16, 0.1), "seq_len"),
        (lambda: mg.decode_attn(q, k, k, pt, idx[:-1], seq, 16, 0.1), "table_idx"),
        (lambda: mg.decode_attn(q, k, k, pt, idx, seq, 16, 0.1, out=q[:-1]), "out"),
        (lambda: mg.decode_attn(q, k[..., :64], k[..., :64], pt, idx, seq, 16, 0.1), "k_cache"),
        (lambda: mg.decode_attn(q, k, k, pt[0], idx, seq, 16, 0.1), "page_table"),
        (lambda: mg.store_decode_attn(q, k[:b], k[:b], idx, k, k[:, :2], pt, idx, seq, 16, 0.1), "v_cache"),
        (lambda: mg.decode_attn_static_workspace(q, k, k, pt, idx, seq, 16, 0.1, out=q[:, :4]), "out"),
        (lambda: mg.extend_attn(q, k, k, pt, idx, seq - 1, seq, idx, 1, 16, 0.1), "q_offset"),
        (lambda: mg.extend_attn(q, k, k, pt, idx, seq[:2] - 1, seq, torch.arange(b + 1, dtype=i32), 1, 16, 0.1),
         "cached_len"),
        (lambda: mg.store_kv(q[0], q[0], idx, k, k), "store_kv"),
    ]
    for call, what in cases:
        with pytest.raises(ValueError, match=what):
            call()
    # right sizes on host memory: refused as not on a CUDA device
    with pytest.raises(ValueError, match="CUDA device"):
        mg.decode_attn(q, k, k, pt, idx, seq, 16, 0.1, num_partitions=4)


def test_binding_shape_checks_accept_what_the_gpu_tests_pass():
    """Every call pattern of the GPU tests, built on host memory, passes the
    binding's shape checks and stops only at the device check."""
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from mg_testlib import GpuStep
    from paged_kv_attention_mg_b200 import workload as wl
    from paged_kv_attention_mg_b200.replicas import shard_kv_heads, take_heads

    def refused_only_for_host_memory(call):
        with pytest.raises(ValueError, match="must be on a CUDA device"):
            call()

    decode_cases = [([5, 9, 12], 16, 8), ([1], 16, 8), ([257, 190], 32, 2), ([130, 7, 400], 28, 4)]
    for lengths, hq, hkv in decode_cases:
        spec = wl.custom_spec("decode", [L - 1 for L in lengths], lengths, hq, hkv, sum(lengths) + 37, seed=1)
        step = wl.make_step(spec)
        g = GpuStep(step, wl.make_layer(step), device="cpu")
        refused_only_for_host_memory(lambda: g.store())
        refused_only_for_host_memory(lambda: g.decode(num_partitions=7))
        refused_only_for_host_memory(lambda: g.store_decode(num_partitions=7))
        refused_only_for_host_memory(lambda: g.extend())  # a decode step as one-token chunks
        refused_only_for_host_memory(lambda: mg.decode_attn_static_workspace(
            g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.seq_len, step.max_seq_len, g.scale,
            num_partitions=7))
        for r in range(2):  # a tensor-parallel rank's slices
            kv0, kv1, q0, q1 = shard_kv_heads(hq, hkv, r, 2)
            refused_only_for_host_memory(lambda: mg.store_decode_attn(
                take_heads(g.q, q0, q1), take_heads(g.k_new, kv0, kv1), take_heads(g.v_new, kv0, kv1), g.out_loc,
                take_heads(g.k_cache, kv0, kv1), take_heads(g.v_cache, kv0, kv1), g.page_table, g.table_idx,
                g.seq_len, step.max_seq_len, g.scale, num_partitions=7))
    extend_cases = [([0], [1], 16, 8), ([130, 0], [300, 257], 16, 8), ([10, 20], [10, 50], 16, 8),
                    ([0, 9], [100, 200], 12, 1)]
    for cached, seq, hq, hkv in extend_cases:
        spec = wl.custom_spec("extend", cached, seq, hq, hkv, sum(seq) + 37, seed=2)
        step = wl.make_step(spec)
        g = GpuStep(step, wl.make_layer(step), device="cpu")
        refused_only_for_host_memory(lambda: g.extend())
        refused_only_for_host_memory(lambda: g.extend(out=torch.empty_like(g.q)))
