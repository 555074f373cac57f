"""GPU: a decode step recorded once into a CUDA graph and replayed over fixed
buffers, as the engine runs decode ("mini-sglang from Scratch Stage 4 ·
Faster and bigger", §What each chapter adds and §Reading these lines: a
captured step needs fixed shapes and fixed buffers, and an input that is not
copied into its buffer gives a silently wrong answer, not an error).

The step is three layers of mg_store_decode_attn (the new token stored into
each layer's pool inside the decode launch).  It is captured with one batch's
inputs in the buffers; then each replay follows a copy of a batch's inputs
into those same buffers -- the first batch again, then a second batch with
other lengths (the launch plan depends only on the max_seq_len hint, so one
capture serves any length mix below it).  Every layer's output is held to the
oracle, and every pool to the host pool after the store, bit for bit.
"""
import pytest
import torch

from mg_testlib import assert_matches_oracle, host_pools_after_store, oracle_decode
from paged_kv_attention_mg_b200 import mg
from paged_kv_attention_mg_b200 import workload as wl

pytestmark = pytest.mark.gpu

LAYERS = 3
HQ, HKV, SLOTS, STRIDE = 32, 8, 12000, 2048


def _batch(lengths, seed):
    spec = wl.custom_spec("decode", [L - 1 for L in lengths], lengths, HQ, HKV, SLOTS, seed, num_layers=LAYERS)
    step = wl.make_step(spec, page_table_stride=STRIDE)
    return step, [wl.make_layer(step, layer) for layer in range(LAYERS)]


class FixedBuffers:
    """The step's device buffers; a batch's inputs are copied into them."""

    def __init__(self, batch):
        dev = "cuda"
        self.q = [torch.empty((batch, HQ, 128), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        self.k_new = [torch.empty((batch, HKV, 128), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        self.v_new = [torch.empty((batch, HKV, 128), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        self.k_cache = [torch.empty((SLOTS, HKV, 128), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        self.v_cache = [torch.empty((SLOTS, HKV, 128), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        self.out = [torch.empty((batch, HQ, 128), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
        self.page_table = torch.empty((batch + 1, STRIDE), dtype=torch.int32, device=dev)
        self.table_idx = torch.empty(batch, dtype=torch.int32, device=dev)
        self.seq_len = torch.empty(batch, dtype=torch.int32, device=dev)
        self.out_loc = torch.empty(batch, dtype=torch.int32, device=dev)
        need = mg.decode_workspace_bytes(batch, HQ, HKV, STRIDE)
        self.workspace = torch.empty(need, dtype=torch.uint8, device=dev)

    def load(self, step, layers):
        """Copy a batch's inputs (metadata, q, new K/V, the pools before the store)."""
        self.page_table.copy_(step.page_table)
        self.table_idx.copy_(step.table_idx)
        self.seq_len.copy_(step.seq_len)
        self.out_loc.copy_(step.out_loc)
        for i, data in enumerate(layers):
            self.q[i].copy_(data.q)
            self.k_new[i].copy_(data.k_new)
            self.v_new[i].copy_(data.v_new)
            self.k_cache[i].copy_(wl.build_pool(step, data.hist_slots, data.k_hist, "cuda"))
            self.v_cache[i].copy_(wl.build_pool(step, data.hist_slots, data.v_hist, "cuda"))

    def run_step(self, scale):
        for i in range(LAYERS):
            mg.store_decode_attn(self.q[i], self.k_new[i], self.v_new[i], self.out_loc, self.k_cache[i],
                                 self.v_cache[i], self.page_table, self.table_idx, self.seq_len, STRIDE, scale,
                                 out=self.out[i], workspace=self.workspace)


def _check(buf, step, layers, what):
    torch.cuda.synchronize()
    assert mg.read_device_error() == 0
    for i, data in enumerate(layers):
        assert_matches_oracle(buf.out[i], oracle_decode(step, data), f"{what}, layer {i}")
        k_ref, v_ref = host_pools_after_store(step, data)
        assert torch.equal(buf.k_cache[i].cpu().view(torch.int16), k_ref.view(torch.int16)), f"{what}: K pool {i}"
        assert torch.equal(buf.v_cache[i].cpu().view(torch.int16), v_ref.view(torch.int16)), f"{what}: V pool {i}"


def test_graph_captured_step_replays_match_the_oracle():
    step_a, layers_a = _batch([1500, 7, 300, 2048, 129, 64], seed=901)
    step_b, layers_b = _batch([20, 1999, 1024, 1, 700, 333], seed=902)
    scale = step_a.spec.scale
    buf = FixedBuffers(step_a.batch)
    buf.load(step_a, layers_a)
    buf.run_step(scale)  # eager warm-up: module load, kernel attributes
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        buf.run_step(scale)
    try:
        buf.load(step_a, layers_a)  # the pools again as before the store
        graph.replay()
        _check(buf, step_a, layers_a, "replay of the captured batch")
        buf.load(step_b, layers_b)  # another batch, other lengths, same buffers
        graph.replay()
        _check(buf, step_b, layers_b, "replay with a second batch copied in")
    finally:
        del graph
