"""Decode without a caller workspace: mg_decode_attn_static_workspace.

Some callers cannot give the library device scratch memory: their device
memory belongs to another allocator (a serving engine's fixed pool, a
framework's caching allocator), they are plug-ins handed only inputs and
outputs, or they run step loops where an allocation (which may synchronise the
device) is not allowed.  For them decode uses a fixed array inside the library.
Here that entry point is checked, through the C ABI, against mg_decode_attn
(which takes the caller's workspace) on two calls in a row.  Both run the same
plan through the same kernels, so their outputs must be identical bit for bit
(any mix-up of the shared array's contents would show); the first call of each
case is also held to the oracle within the tolerance every decode test uses.
The file name makes pytest collect it last, so if it fails, a run that stops
at the first failure has run everything else.
"""
import pytest
import torch

from mg_testlib import GpuStep, assert_matches_oracle, oracle_decode
from paged_kv_attention_mg_b200 import mg
from paged_kv_attention_mg_b200 import workload as wl

pytestmark = pytest.mark.gpu


def _identical(got: torch.Tensor, ref: torch.Tensor, what: str):
    assert torch.isfinite(got.float()).all(), what
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), (
        f"{what}: {int((got.view(torch.int16) != ref.view(torch.int16)).sum())} elements differ, "
        f"max |diff| {float((got.float() - ref.float()).abs().max()):.3e}")


def _decode_static(g: GpuStep, parts: int = 0):
    return mg.decode_attn_static_workspace(g.q, g.k_cache, g.v_cache, g.page_table, g.table_idx, g.seq_len,
                                           g.step.max_seq_len, g.scale, num_partitions=parts)


def _cases():
    spec = wl.BY_NAME["qwen3_0.6b_decode_28l"]
    step = wl.make_step(spec)
    yield "qwen3 layer 0", step, wl.make_layer(step, 0), 0, [0, 17, 63]
    lengths = [700, 3, 1500, 64, 2049]
    spec = wl.custom_spec("decode", [L - 1 for L in lengths], lengths, 32, 8, sum(lengths) + 100, seed=77)
    step = wl.make_step(spec)
    yield "group 4, forced partitions", step, wl.make_layer(step), 37, None


def test_static_workspace_matches_caller_workspace_on_two_calls():
    cases = []
    for name, step, data, parts, sample in _cases():
        g = GpuStep(step, data)
        g.store()
        ref = g.decode(num_partitions=parts)  # the entry point with a caller workspace
        cases.append((name, step, data, g, parts, sample, ref))
    # two calls in a row for each case, interleaved so each call follows one
    # that left other contents in the shared array
    for call in range(2):
        for name, step, data, g, parts, sample, ref in cases:
            out = _decode_static(g, parts)
            _identical(out, ref, f"{name}, call {call + 1}")
            if call == 0:
                assert_matches_oracle(out, oracle_decode(step, data, requests=sample), f"{name} vs the oracle")
    assert mg.read_device_error() == 0


def test_static_workspace_refuses_a_plan_beyond_its_size():
    b, hq, hkv, d = 4096, 128, 8, 128  # partial slots for 4096 x 8 pairs: far beyond 16 MiB
    need = mg.decode_workspace_bytes(b, hq, hkv, 16)
    assert need > mg.STATIC_WORKSPACE_BYTES
    q = torch.zeros((b, hq, d), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((64, hkv, d), dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros((b + 1, 32), dtype=torch.int32, device="cuda")
    idx = torch.arange(b, dtype=torch.int32, device="cuda")
    seq = torch.ones(b, dtype=torch.int32, device="cuda")
    with pytest.raises(mg.MgError) as e:
        mg.decode_attn_static_workspace(q, pool, pool, pt, idx, seq, 16, 0.1)
    assert e.value.status == 4  # MG_ERR_WORKSPACE_TOO_SMALL, refused before any launch
