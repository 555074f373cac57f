#!/usr/bin/env python
"""Benchmark of the paged KV attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the hot path over one batch: for the default workload
(Qwen3-0.6B attention shape, 28 layers, batch 64, lengths U[128, 2048]) that
is, for every layer, the KV store of the 64 new tokens into that layer's pool
followed by paged decode attention over the page table.  Each layer has its
own 200k-slot pool, so a step reads ~7.3 GB of KV: inputs larger than L2, no
flush needed.  With N GPUs every rank runs its own replica with its own seed
(weak scaling, no collective on the data path); the reported time is the max
over ranks.

The step is recorded once into a CUDA graph over fixed buffers and replayed,
as the engine runs decode (--no-graph launches it eagerly instead).

The JSON line: `value` = algorithmic bytes (K/V rows once per GQA group, q,
out, page-table entries, plus the store's reads and writes) per step summed
over ranks / step time, in GB/s; `e2e` = the same through the public API with
the step's inputs copied from pinned host memory into the fixed buffers and
the outputs copied back inside the timed region (two buffer sets in turn, so
a step's host copies, on two copy streams, overlap the neighbouring steps'
layer calls, as a serving loop's would); `roofline` = one layer's
mg_store_decode_attn call (decode kernel with the store fused, then the merge
kernel; --unfused: mg_decode_attn after a separate mg_store_kv) against the
measured HBM copy bandwidth, its duration the timed step's device time over
the layer calls it holds (the decode step's graph holds nothing else), with
the DRAM bytes per launch ncu measured for these kernel sources
(profiles/traffic.json); `call_us_events` is the same call timed by events
recorded around every call inside a second, instrumented copy of the step
(each event node ends the programmatic overlap of the next call's launch, so
it reads a few microseconds longer); `cpu_baseline` = the fp64 oracle on this
host's cores on a bounded sample of the same workload.  --workload
chunked_prefill_extend measures extend (TFLOP/s against the dense bf16 peak).

--impl reference times the oracle itself (there is no other implementation
of this path to run) on the same metric, rank 0 only.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from paged_kv_attention_mg_b200 import roofline as rf  # noqa: E402
from paged_kv_attention_mg_b200.replicas import Replicas, rank_spec  # noqa: E402
from paged_kv_attention_mg_b200 import workload as wl  # noqa: E402

METRIC = "paged decode-attention KV GB/s (% of HBM peak) and decode tokens/s, 1 B200"
EXTEND_METRIC = "chunked-prefill extend attention TFLOP/s (unmasked QK^T + PV flops), 1 B200"
L2_BYTES = 126 * 1024 * 1024  # B200 L2; a decode step reading less than 4x this is timed with an L2 flush
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ["include/mg.h", "paged_kv_attention_mg_b200/csrc/mg.cu",
                  "paged_kv_attention_mg_b200/csrc/common.cuh", "paged_kv_attention_mg_b200/csrc/ptx.cuh",
                  "paged_kv_attention_mg_b200/csrc/store_kv.cuh", "paged_kv_attention_mg_b200/csrc/decode.cuh",
                  "paged_kv_attention_mg_b200/csrc/extend.cuh"]


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3_0.6b_decode_28l", choices=sorted(wl.BY_NAME))
    ap.add_argument("--partitions", type=int, default=0, help="decode workers (0 = automatic plan)")
    ap.add_argument("--extend-ctas", type=int, default=-1,
                    help="mixed batches: SMs for the extend kernel beside the decode kernel "
                         "(-1 = mg.mixed_extend_ctas's estimate, 0 = one kernel after the other)")
    ap.add_argument("--layers", type=int, default=0,
                    help="run only the first N layers (small cases for profiling; 0 = the workload's own)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every step eagerly instead of a CUDA graph")
    ap.add_argument("--unfused", action="store_true", help="separate KV-store launch before each decode")
    ap.add_argument("--plain", action="store_true",
                    help="shared-prefix workloads: plain mg_decode_attn over the same shared page tables "
                         "(every request reads the prefix), for comparison with the shared-prefix decode")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="bound of the cpu_baseline sample")
    ap.add_argument("--cpu-seconds-1thread", type=float, default=8.0,
                    help="bound of the cpu_baseline's one-thread sample (0 skips it)")
    ap.add_argument("--soak-seconds", type=float, default=1.5,
                    help="extra untimed warm-up so the clock sampler sees the GPU under load")
    return ap.parse_args()


# ----------------------------------------------------------------------------- plumbing

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), float(m.get("bf16_tflops_sustained", 0)), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def _code_only(src: str) -> str:
    """C/C++ source without its comments and with whitespace collapsed, so that
    editing a comment does not change the digest of the kernels (string
    literals are kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"':  # string literal
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_digest() -> str:
    """Digest of the kernel sources' code (comments and layout excluded): the
    key under which profiles/traffic.json holds measured DRAM bytes."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary,
    or None if there is none or the kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entries = json.load(f)
    e = entries.get(workload)
    if not e or e.get("source_digest") != source_digest():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        sel = []
        try:
            bus = torch.cuda.get_device_properties(device_index).pci_bus_id
            sel = ["-i", f"{torch.cuda.get_device_properties(device_index).pci_domain_id:08x}:{bus:02x}:"
                   f"{torch.cuda.get_device_properties(device_index).pci_device_id:02x}.0"]
        except Exception:
            sel = []
        self.sel = sel

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [ln.strip().split(",") for ln in self.file.read().splitlines() if ln.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- workloads

def make_layers(step, num_layers, device):
    """Per-layer device tensors.  Host generation runs on a thread pool (each
    layer has its own generator, so the result does not depend on threading)."""
    def one(layer):
        data = wl.make_layer(step, layer)
        k = wl.build_pool(step, data.hist_slots, data.k_hist, device)
        v = wl.build_pool(step, data.hist_slots, data.v_hist, device)
        return dict(q=data.q.to(device), k_new=data.k_new.to(device), v_new=data.v_new.to(device),
                    k_cache=k, v_cache=v, q_host=data.q, k_new_host=data.k_new, v_new_host=data.v_new)
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        return list(ex.map(one, range(num_layers)))


def pack_io(bench, out_shape):
    """Place the step's per-layer inputs (q, k_new, v_new) in one contiguous
    device buffer and the per-layer outputs in another, each mirrored by one
    pinned host buffer, so the end-to-end step moves them with one copy each
    way.  The layers' tensors become views into these buffers."""
    names = ("q", "k_new", "v_new")
    sizes = [bench.layers[0][n].numel() for n in names]
    per = sum(sizes)
    L = len(bench.layers)
    bench.in_dev = torch.empty(L * per, dtype=torch.bfloat16, device=bench.device)
    bench.in_host = torch.empty(L * per, dtype=torch.bfloat16, pin_memory=True)
    for i, lay in enumerate(bench.layers):
        off = i * per
        for n, sz in zip(names, sizes):
            shape = lay[n].shape
            view = bench.in_dev[off:off + sz].view(shape)
            view.copy_(lay[n])
            bench.in_host[off:off + sz].view(shape).copy_(lay.pop(n + "_host"))
            lay[n] = view
            off += sz
    per_out = math.prod(out_shape)
    bench.out_dev = torch.empty(L * per_out, dtype=torch.bfloat16, device=bench.device)
    bench.out_host = torch.empty(L * per_out, dtype=torch.bfloat16, pin_memory=True)
    bench.outs = [bench.out_dev[i * per_out:(i + 1) * per_out].view(out_shape) for i in range(L)]


def io_bytes(bench):
    """Bytes the end-to-end step copies host -> device and device -> host."""
    h2d = sum(t.numel() * t.element_size() for t in bench.meta_host.values())
    h2d += bench.in_host.numel() * bench.in_host.element_size()
    return h2d, bench.out_host.numel() * bench.out_host.element_size()


class IoSet:
    """One of the two buffer sets an end-to-end step alternates between: device
    copies of the step's inputs (metadata, every layer's q / k / v rows) and
    outputs, a pinned host buffer for the outputs, the layers' views into them,
    and the events that order its copies and its layer calls."""

    def __init__(self, bench, first: bool):
        if first:  # the buffers the bench already holds
            self.in_dev, self.out_dev, self.meta = bench.in_dev, bench.out_dev, bench.meta
            self.layers, self.outs = bench.layers, bench.outs
            self.out_host = bench.out_host
        else:
            self.in_dev = bench.in_dev.clone()
            self.out_dev = torch.empty_like(bench.out_dev)
            self.out_host = torch.empty_like(bench.out_host).pin_memory()
            self.meta = {n: t.clone() for n, t in bench.meta.items()}
            base, es = bench.in_dev.data_ptr(), bench.in_dev.element_size()

            def view(t):  # the same view of this set's input buffer
                off = (t.data_ptr() - base) // es
                return self.in_dev[off:off + t.numel()].view(t.shape)
            self.layers = [dict(lay, q=view(lay["q"]), k_new=view(lay["k_new"]), v_new=view(lay["v_new"]))
                           for lay in bench.layers]
            per = bench.out_dev.numel() // len(bench.layers)
            self.outs = [self.out_dev[i * per:(i + 1) * per].view(o.shape) for i, o in enumerate(bench.outs)]
        self.in_done, self.compute_done, self.out_done = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
        self.run = None

    def compute(self, bench):
        for i, lay in enumerate(self.layers):
            bench.layer(lay, self.outs[i], self.meta)


def pipelined_io_step(bench, io, side_in, side_out):
    """One end-to-end step on buffer set `io`: its inputs copied from pinned host
    memory on a copy stream, its layer calls, its outputs copied back on a
    second copy stream.  Consecutive steps use the two sets in turn, so a
    step's copies overlap its neighbours' layers, as a serving loop's would;
    each set's copies wait for the last use of the buffers they overwrite."""
    main = torch.cuda.current_stream()
    side_in.wait_event(io.compute_done)  # the previous step on this set has read its inputs
    with torch.cuda.stream(side_in):
        for n, t in bench.meta_host.items():
            io.meta[n].copy_(t, non_blocking=True)
        io.in_dev.copy_(bench.in_host, non_blocking=True)
        io.in_done.record(side_in)
    main.wait_event(io.in_done)
    main.wait_event(io.out_done)  # ... and its outputs have left the device
    io.run()
    io.compute_done.record(main)
    side_out.wait_event(io.compute_done)
    with torch.cuda.stream(side_out):
        io.out_host.copy_(io.out_dev, non_blocking=True)
        io.out_done.record(side_out)


class DecodeBench:
    def __init__(self, spec, step, device, partitions, fused=True, plain=False, extend_ctas=-1):
        from paged_kv_attention_mg_b200 import mg
        self.mg = mg
        self.fused = fused
        self.spec, self.step, self.device = spec, step, device
        self.layers = make_layers(step, spec.num_layers, device)
        # shared-prefix workloads: groups of requests read their common prefix once
        # (mg_store_decode_attn_shared_prefix; --unfused: mg_store_kv, then
        # mg_decode_attn_shared_prefix; --plain: the plain decode over the same tables)
        self.shared = step.group_first is not None and not plain
        self.fused = fused
        names = ("page_table", "table_idx", "seq_len", "out_loc") + (("group_first", "prefix_len") if self.shared
                                                                      else ())
        self.meta = {n: getattr(step, n).to(device) for n in names}
        self.meta_host = {n: getattr(step, n).pin_memory() for n in names}
        self.max_seq_len = step.max_seq_len
        self.partitions = partitions
        B, hq, hkv = step.batch, spec.num_q_heads, spec.num_kv_heads
        self.workers, self.slots = mg.decode_plan(B, hkv, self.max_seq_len, partitions)
        if self.shared:
            ng = int(step.prefix_len.numel())
            ws = mg.decode_shared_prefix_workspace_bytes(B, ng, hq, hkv, self.max_seq_len, partitions)
        else:
            ws = mg.decode_workspace_bytes(B, hq, hkv, self.max_seq_len, partitions)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)
        pack_io(self, (B, hq, spec.head_dim))
        L = step.seq_len.tolist()
        if step.group_first is not None:  # the prefix counted once, whichever kernel reads it
            self.decode_bytes = rf.decode_bytes_shared_prefix(L, step.group_first.tolist(), step.prefix_len.tolist(),
                                                              hq, hkv, spec.head_dim)
        else:
            self.decode_bytes = rf.decode_bytes(L, hq, hkv, spec.head_dim)
        self.store_bytes = rf.store_bytes(step.num_new_tokens, hkv, spec.head_dim)
        self.step_bytes = spec.num_layers * (self.decode_bytes + self.store_bytes)
        self.tokens_per_step = B
        # per layer: (store,) decode workers, merge
        self.launches_per_step = spec.num_layers * (2 if self.fused else 3)
        # what one timed layer call moves: the store and the decode (fused or not;
        # the call's duration is the step time over its layer calls)
        self.kernel_bytes = self.decode_bytes + self.store_bytes
        self.h2d_bytes, self.d2h_bytes = io_bytes(self)
        self.ev = None

    def layer(self, lay, out, meta, events=None):
        mg = self.mg
        if self.shared and self.fused:
            if events:
                events[0].record()
            mg.store_decode_attn_shared_prefix(lay["q"], lay["k_new"], lay["v_new"], meta["out_loc"],
                                               lay["k_cache"], lay["v_cache"], meta["page_table"],
                                               meta["table_idx"], meta["seq_len"], meta["group_first"],
                                               meta["prefix_len"], self.max_seq_len, self.spec.scale,
                                               num_partitions=self.partitions, out=out, workspace=self.workspace)
            if events:
                events[1].record()
            return
        if self.shared:
            mg.store_kv(lay["k_new"], lay["v_new"], meta["out_loc"], lay["k_cache"], lay["v_cache"])
            if events:
                events[0].record()
            mg.decode_attn_shared_prefix(lay["q"], lay["k_cache"], lay["v_cache"], meta["page_table"],
                                         meta["table_idx"], meta["seq_len"], meta["group_first"],
                                         meta["prefix_len"], self.max_seq_len, self.spec.scale,
                                         num_partitions=self.partitions, out=out, workspace=self.workspace)
            if events:
                events[1].record()
            return
        if self.fused:  # store + decode in one decode launch
            if events:
                events[0].record()
            mg.store_decode_attn(lay["q"], lay["k_new"], lay["v_new"], meta["out_loc"], lay["k_cache"],
                                 lay["v_cache"], meta["page_table"], meta["table_idx"], meta["seq_len"],
                                 self.max_seq_len, self.spec.scale, num_partitions=self.partitions, out=out,
                                 workspace=self.workspace)
            if events:
                events[1].record()
            return
        mg.store_kv(lay["k_new"], lay["v_new"], meta["out_loc"], lay["k_cache"], lay["v_cache"])
        if events:
            events[0].record()
        mg.decode_attn(lay["q"], lay["k_cache"], lay["v_cache"], meta["page_table"], meta["table_idx"],
                       meta["seq_len"], self.max_seq_len, self.spec.scale, num_partitions=self.partitions, out=out,
                       workspace=self.workspace)
        if events:
            events[1].record()

    def run_step(self, events=None):
        for i, lay in enumerate(self.layers):
            self.layer(lay, self.outs[i], self.meta, events[i] if events else None)

    def kernel_bytes(self):
        return self.decode_bytes

    def details(self):
        d = {"decode_workers": self.workers, "store": "fused into decode" if self.fused else "separate launch"}
        if self.step.group_first is not None:
            d["shared_prefix"] = {"read": "once per group (mg_decode_attn_shared_prefix)" if self.shared
                                  else "by every request (mg_decode_attn over the same page tables)",
                                  "groups": int(self.step.prefix_len.numel()),
                                  "prefix_len": sorted(set(self.step.prefix_len.tolist())),
                                  "bytes_if_unshared": rf.decode_bytes(self.step.seq_len.tolist(),
                                                                       self.spec.num_q_heads, self.spec.num_kv_heads,
                                                                       self.spec.head_dim)}
        return d


class ExtendBench:
    def __init__(self, spec, step, device, partitions, fused=True, plain=False, extend_ctas=-1):
        from paged_kv_attention_mg_b200 import mg
        self.mg = mg
        self.spec, self.step, self.device = spec, step, device
        self.layers = make_layers(step, spec.num_layers, device)
        names = ("page_table", "table_idx", "seq_len", "cached_len", "q_offset", "out_loc")
        self.meta = {n: getattr(step, n).to(device) for n in names}
        self.meta_host = {n: getattr(step, n).pin_memory() for n in names}
        pack_io(self, tuple(self.layers[0]["q"].shape))
        c, s = step.cached_len.tolist(), step.seq_len.tolist()
        self.flops = rf.extend_flops(c, s, spec.num_q_heads, spec.head_dim)
        self.extend_bytes = rf.extend_bytes(c, s, spec.num_q_heads, spec.num_kv_heads, spec.head_dim)
        self.store_bytes = rf.store_bytes(step.num_new_tokens, spec.num_kv_heads, spec.head_dim)
        self.tokens_per_step = step.num_new_tokens
        # a mixed batch runs through mg_mixed_attn: store, decode workers, merge, extend
        self.mixed = spec.mixed
        self.launches_per_step = spec.num_layers * (4 if self.mixed else 2)
        self.h2d_bytes, self.d2h_bytes = io_bytes(self)
        self.workers = None
        self.extend_ctas = 0
        if self.mixed:
            ws = mg.mixed_workspace_bytes(step.batch, spec.num_q_heads, spec.num_kv_heads, step.max_seq_len, partitions)
            self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)
            self.workers, _ = mg.decode_plan(step.batch, spec.num_kv_heads, step.max_seq_len, partitions)
            sms = torch.cuda.get_device_properties(device).multi_processor_count
            self.extend_ctas = (mg.mixed_extend_ctas(c, s, spec.num_q_heads, spec.num_kv_heads, sms)
                                if extend_ctas < 0 else extend_ctas)
            if self.extend_ctas > 0:  # the decode kernel's workers on the SMs left to it
                per_sm = mg.decode_plan(step.batch, spec.num_kv_heads, step.max_seq_len, 0)[0] // sms
                w = per_sm * (sms - min(self.extend_ctas, sms - 1))
                self.workers, _ = mg.decode_plan(step.batch, spec.num_kv_heads, step.max_seq_len,
                                                 partitions if 0 < partitions < w else w)
        self.partitions = partitions

    def layer(self, lay, out, meta, events=None):
        mg, st = self.mg, self.step
        mg.store_kv(lay["k_new"], lay["v_new"], meta["out_loc"], lay["k_cache"], lay["v_cache"])
        if events:
            events[0].record()
        if self.mixed:
            mg.mixed_attn(lay["q"], lay["k_cache"], lay["v_cache"], meta["page_table"], meta["table_idx"],
                          meta["cached_len"], meta["seq_len"], meta["q_offset"], st.max_q_len, st.max_seq_len,
                          self.spec.scale, num_partitions=self.partitions, extend_ctas=self.extend_ctas, out=out,
                          workspace=self.workspace)
        else:
            mg.extend_attn(lay["q"], lay["k_cache"], lay["v_cache"], meta["page_table"], meta["table_idx"],
                           meta["cached_len"], meta["seq_len"], meta["q_offset"], st.max_q_len, st.max_seq_len,
                           self.spec.scale, out=out)
        if events:
            events[1].record()

    run_step = DecodeBench.run_step

    def details(self):
        d = {"kv_bytes_per_step": self.extend_bytes}
        if self.mixed:
            d.update({"entry_point": "mg_mixed_attn (one-token requests: decode kernel + merge; chunks: extend kernel)",
                      "decode_workers": self.workers, "extend_ctas": self.extend_ctas})
        return d


def decode_needs_flush(spec, step) -> bool:
    """A decode step whose K/V reads are under 4x the L2 is timed with an L2
    flush between steps (larger ones stream past the L2 by themselves)."""
    if step.group_first is not None:
        per_layer = rf.decode_bytes_shared_prefix(step.seq_len.tolist(), step.group_first.tolist(),
                                                  step.prefix_len.tolist(), spec.num_q_heads, spec.num_kv_heads,
                                                  spec.head_dim)
    else:
        per_layer = rf.decode_bytes(step.seq_len.tolist(), spec.num_q_heads, spec.num_kv_heads, spec.head_dim)
    return spec.num_layers * per_layer < 4 * L2_BYTES


def workload_config(spec, step, n_gpus: int) -> dict:
    """The `config` of the JSON line: the workload and how it is run, the same
    for this library's arm and the reference arm."""
    common = {"workload": spec.name, "batch": step.batch, "layers": spec.num_layers, "q_heads": spec.num_q_heads,
              "kv_heads": spec.num_kv_heads, "head_dim": spec.head_dim, "pool_slots": spec.num_slots}
    if spec.kind == "decode":
        if step.group_first is not None:
            per_layer = rf.decode_bytes_shared_prefix(step.seq_len.tolist(), step.group_first.tolist(),
                                                      step.prefix_len.tolist(), spec.num_q_heads,
                                                      spec.num_kv_heads, spec.head_dim)
        else:
            per_layer = rf.decode_bytes(step.seq_len.tolist(), spec.num_q_heads, spec.num_kv_heads, spec.head_dim)
        common.update({"mean_seq_len": round(float(step.seq_len.double().mean()), 1),
                       "max_seq_len": step.max_seq_len})
        if decode_needs_flush(spec, step):
            common["l2"] = (f"L2 flushed between timed steps (256 MB write): {per_layer / 1e6:.0f} MB read per "
                            f"step, under 4x the L2")
        else:
            common["l2"] = (f"inputs larger than L2: {spec.num_layers} per-layer pools, "
                            f"{spec.num_layers * per_layer / 1e9:.2f} GB read per step")
    else:
        n = step.seq_len - step.cached_len
        common.update({"new_tokens": int(n.sum()), "mean_cached_len": round(float(step.cached_len.double().mean()), 1),
                       "l2": "L2 flushed between timed steps (256 MB write)"})
    common["parallelism"] = f"dp{n_gpus} (independent replicas, no collective)" if n_gpus > 1 else "single GPU"
    return common


# ----------------------------------------------------------------------------- cpu baseline

class OracleSampler:
    """The oracle timed on bounded samples of the workload on the host cores.

    Inputs are generated once and held across samples (decode: at most
    `max_layers` distinct layers, each a full pool; extend: one layer), so a
    sample times the oracle and not the synthetic-input generator.  A decode
    sample runs whole layer calls (all requests), an extend sample whole
    requests in turn, until `seconds` of oracle time are spent."""

    def __init__(self, spec, step, threads: int, max_layers: int = 2):
        self.spec, self.step, self.threads = spec, step, threads
        self.max_layers = max(1, min(max_layers, spec.num_layers))
        self._layers = []
        self._next = 0  # decode: next cached layer; extend: next request

    def _inputs(self, layer: int):
        while len(self._layers) <= layer:
            step = self.step
            data = wl.make_layer(step, len(self._layers))
            k = wl.build_pool(step, data.hist_slots, data.k_hist)
            v = wl.build_pool(step, data.hist_slots, data.v_hist)
            loc = step.out_loc.to(torch.int64)
            k.index_copy_(0, loc, data.k_new)
            v.index_copy_(0, loc, data.v_new)
            self._layers.append((wl.bits(data.q), wl.bits(k), wl.bits(v)))
        return self._layers[layer]

    def sample(self, seconds: float):
        """Returns (bytes_or_flops, oracle seconds, what the sample was, unit)."""
        import oracle
        spec, step = self.spec, self.step
        work, total_t, calls = 0, 0.0, 0
        if spec.kind == "decode":
            if step.group_first is not None:  # the same algorithmic bytes as the GPU arm: a shared prefix once
                per_layer = rf.decode_bytes_shared_prefix(step.seq_len.tolist(), step.group_first.tolist(),
                                                          step.prefix_len.tolist(), spec.num_q_heads,
                                                          spec.num_kv_heads, spec.head_dim)
            else:
                per_layer = rf.decode_bytes(step.seq_len.tolist(), spec.num_q_heads, spec.num_kv_heads,
                                            spec.head_dim)
            while calls == 0 or total_t < seconds:
                q, k, v = self._inputs(self._next)
                self._next = (self._next + 1) % self.max_layers
                t0 = time.perf_counter()
                oracle.decode(q, k, v, step.page_table.numpy(), step.table_idx.numpy(), step.seq_len.numpy(),
                              spec.scale, threads=self.threads)
                total_t += time.perf_counter() - t0
                work += per_layer
                calls += 1
            return (work, total_t, f"{calls} layer calls (all {step.batch} requests each) over "
                    f"{len(self._layers)} generated layers", "GB/s")
        q, k, v = self._inputs(0)
        c, s = step.cached_len.tolist(), step.seq_len.tolist()
        while calls == 0 or total_t < seconds:
            r = self._next
            self._next = (self._next + 1) % step.batch
            t0 = time.perf_counter()
            oracle.extend(q, k, v, step.page_table.numpy(), step.table_idx.numpy(), step.cached_len.numpy(),
                          step.seq_len.numpy(), step.q_offset.numpy(), spec.scale, requests=[r],
                          threads=self.threads)
            total_t += time.perf_counter() - t0
            work += rf.extend_flops([c[r]], [s[r]], spec.num_q_heads, spec.head_dim)
            calls += 1
        return work, total_t, f"{calls} requests of one layer (of {step.batch}, taken in turn)", "TFLOP/s"


def cpu_model() -> str:
    """The host CPU's model name (first processor in /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(spec, step, seconds: float, seconds_1thread: float) -> dict:
    """The oracle on this host: all cores (the reported value), then one thread."""
    threads = cpu_threads()
    w, secs, sample, unit = OracleSampler(spec, step, threads).sample(seconds)
    scale = 1e9 if unit == "GB/s" else 1e12
    line = {"value": round(w / secs / scale, 4), "unit": unit, "cores": threads, "kind": "oracle",
            "sample": sample, "seconds": round(secs, 2), "cpu_model": cpu_model()}
    if seconds_1thread > 0:
        w1, s1, sample1, _ = OracleSampler(spec, step, 1).sample(seconds_1thread)
        line.update({"value_1thread": round(w1 / s1 / scale, 4), "sample_1thread": sample1,
                     "seconds_1thread": round(s1, 2)})
    return line


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    """The oracle as the reference arm: rank 0 only, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    spec = wl.BY_NAME[args.workload]
    step = wl.make_step(spec)
    threads = cpu_threads()
    per_step_seconds = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    sampler = OracleSampler(spec, step, threads)
    for _ in range(args.warmup):
        sampler.sample(per_step_seconds)
    work, secs = 0, 0.0
    sample = unit = None
    for _ in range(args.steps):
        w, t, sample, unit = sampler.sample(per_step_seconds)
        work += w
        secs += t
    value = (work / secs / 1e9) if unit == "GB/s" else (work / secs / 1e12)
    line = {"impl": "reference", "metric": METRIC if spec.kind == "decode" else EXTEND_METRIC,
            "value": round(value, 4), "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(spec, step, args.gpus), "arm": "oracle on the host cores",
            "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": threads, "kind": "oracle",
                             "sample": f"per step: {sample}"},
            "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    dist = Replicas(args.gpus, backend="nccl")
    device = torch.device("cuda", dist.local)
    torch.cuda.set_device(device)
    spec = rank_spec(wl.BY_NAME[args.workload], dist.rank)
    if args.layers:
        spec = dataclasses.replace(spec, num_layers=min(args.layers, spec.num_layers))
    step = wl.make_step(spec)
    bench = (DecodeBench if spec.kind == "decode" else ExtendBench)(spec, step, device, args.partitions,
                                                                     fused=not args.unfused, plain=args.plain,
                                                                     extend_ctas=args.extend_ctas)
    flush = None
    if spec.kind == "extend" or decode_needs_flush(spec, step):
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    torch.cuda.synchronize()

    # The step as the engine runs decode: recorded once into a CUDA graph over
    # fixed buffers, then replayed (--no-graph: launched eagerly every step).
    # Timing events around every attention call are recorded inside the step
    # (graph-capturable "external" events), so the kernel time is measured in
    # the timed region itself, free of host launch gaps.
    use_graph = not args.no_graph
    kev = [(torch.cuda.Event(enable_timing=True, external=use_graph),
            torch.cuda.Event(enable_timing=True, external=use_graph)) for _ in range(spec.num_layers)]
    fev = (torch.cuda.Event(enable_timing=True, external=use_graph),
           torch.cuda.Event(enable_timing=True, external=use_graph))

    def enqueue_step():
        if flush is not None:
            fev[0].record()
            flush.fill_(0x5A)
            fev[1].record()
        bench.run_step(kev)

    for _ in range(2):  # eager warm-up: module load, kernel attributes
        enqueue_step()
    torch.cuda.synchronize()
    graphs = []
    if use_graph:
        g_timed, g_plain = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_timed):
            enqueue_step()
        with torch.cuda.graph(g_plain):
            bench.run_step()
        graphs = [g_timed, g_plain]
        run_timed, run_plain = g_timed.replay, g_plain.replay
    else:
        run_timed, run_plain = enqueue_step, bench.run_step
    torch.cuda.synchronize()

    # The decode step holds only the layer calls, so it is timed without
    # instrumentation and a call's duration is the step time over its calls;
    # the instrumented copy is replayed afterwards for the per-call events.
    # The extend step also holds the L2 flush, timed by its own events and
    # taken out, so that step runs instrumented.
    run_step = run_plain if flush is None else run_timed
    sampler = ClockSampler(dist.local)
    sampler.start()
    # warm-up (W steps) plus a short soak so clocks are sampled under load
    for _ in range(max(3, args.warmup)):
        run_step()
    torch.cuda.synchronize()
    t_end = time.perf_counter() + args.soak_seconds
    while time.perf_counter() < t_end:
        for _ in range(10):
            run_step()
        torch.cuda.synchronize()

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for _ in range(args.steps):
        run_step()
    stop.record()
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop()
    total_ms = start.elapsed_time(stop)
    flush_ms = fev[0].elapsed_time(fev[1]) if flush is not None else 0.0  # last step's flush
    step_ms_local = total_ms / args.steps - flush_ms
    if spec.kind == "decode":
        kernel_ms_local = step_ms_local / spec.num_layers
        for _ in range(3):  # the instrumented copy, outside the timed region
            run_timed()
        torch.cuda.synchronize()
    else:
        kernel_ms_local = None
    events_ms_local = sum(a.elapsed_time(b) for a, b in kev) / spec.num_layers  # last step's calls
    if kernel_ms_local is None:
        kernel_ms_local = events_ms_local
    step_ms = dist.max(step_ms_local)
    kernel_ms = dist.max(kernel_ms_local)
    events_ms = dist.max(events_ms_local)
    # the roofline is per GPU: every rank's own work over its own call time (ranks
    # draw their own lengths), and the line reports the lowest rank's figure
    local_work = bench.kernel_bytes if spec.kind == "decode" else bench.flops
    achieved_local = local_work / (kernel_ms_local * 1e-3) / (1e9 if spec.kind == "decode" else 1e12)
    achieved_min = dist.min(achieved_local)
    # every rank draws its own lengths, so the job's work per step is the sum over ranks
    step_work = dist.sum(float(bench.step_bytes if spec.kind == "decode" else bench.flops))
    step_tokens = dist.sum(float(bench.tokens_per_step))
    h2d_bytes = int(dist.sum(float(bench.h2d_bytes)))
    d2h_bytes = int(dist.sum(float(bench.d2h_bytes)))

    # end to end through the public API with host buffers: this step's inputs
    # copied from pinned host memory into the fixed device buffers, the step,
    # the outputs copied back to pinned host memory
    e2e = None
    if not args.no_e2e:
        side_in, side_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        sets = [IoSet(bench, True), IoSet(bench, False)]
        for io in sets:
            if use_graph:  # each set's layer calls as one graph, like the timed step
                io.compute(bench)
                torch.cuda.synchronize()
                g_io = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g_io):
                    io.compute(bench)
                graphs.append(g_io)
                io.run = g_io.replay
            else:
                io.run = (lambda io=io: io.compute(bench))
        torch.cuda.synchronize()
        for k in range(4):
            pipelined_io_step(bench, sets[k & 1], side_in, side_out)
        torch.cuda.synchronize()
        dist.barrier()
        main = torch.cuda.current_stream()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps = max(3, args.steps)
        ea.record()
        for k in range(e2e_steps):
            pipelined_io_step(bench, sets[k & 1], side_in, side_out)
        main.wait_stream(side_out)
        main.wait_stream(side_in)
        eb.record()
        torch.cuda.synchronize()
        e2e = dist.max(ea.elapsed_time(eb) / e2e_steps)

    hbm, tflops, tflops_sus, peak_src = measured_peaks()
    n = args.gpus
    if spec.kind == "decode":
        value = step_work / (step_ms * 1e-3) / 1e9
        unit = "GB/s"
        metric = METRIC
        achieved = achieved_min
        kname = ("decode_kernel<shared prefix, fused store> + decode_merge_kernel (one "
                 "mg_store_decode_attn_shared_prefix call)" if bench.shared and bench.fused
                 else "store_kv_kernel + decode_kernel<shared prefix> + decode_merge_kernel (mg_store_kv + "
                      "mg_decode_attn_shared_prefix)" if bench.shared
                 else "decode_kernel<fused store> + decode_merge_kernel (one mg_store_decode_attn call)" if bench.fused
                 else "store_kv_kernel + decode_kernel + decode_merge_kernel (mg_store_kv + mg_decode_attn)")
        roof = {"bound": "hbm", "kernel": kname,
                "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "peak_source": f"{peak_src} HBM copy bandwidth",
                "call_us": round(kernel_ms * 1e3, 3), "duration": "timed step / layer calls in it",
                "call_us_events": round(events_ms * 1e3, 3),
                "traffic": profiled_traffic(spec.name + (":plain" if args.plain else ""))}
        extra = {"tokens_per_s": round(step_tokens / (step_ms * 1e-3), 1),
                 "frac_of_8tbs_nominal": round(value / n / 8000.0, 4),
                 "frac_of_measured_hbm": round(value / n / hbm, 4)}
    else:
        value = step_work / (step_ms * 1e-3) / 1e12
        unit = "TFLOP/s"
        metric = EXTEND_METRIC
        achieved = achieved_min
        # the call's bound: tensor cores for its unmasked flops, or HBM for its K/V
        # bytes (a batch of mostly decode requests), whichever takes longer at peak
        kv_gbs = bench.extend_bytes / (kernel_ms_local * 1e-3) / 1e9
        if bench.extend_bytes / (hbm * 1e9) > bench.flops / (tflops * 1e12):
            kname = ("decode_kernel + decode_merge_kernel + extend_kernel (one mg_mixed_attn call)" if bench.mixed
                     else "extend_kernel")
            roof = {"bound": "hbm", "kernel": kname, "achieved": round(kv_gbs, 1), "peak": hbm,
                    "unit": "GB/s", "frac": round(kv_gbs / hbm, 4), "peak_source": f"{peak_src} HBM copy bandwidth",
                    "tflops": round(achieved, 1), "traffic": profiled_traffic(spec.name)}
        else:
            roof = {"bound": "tensor", "kernel": "extend_kernel", "achieved": round(achieved, 1), "peak": tflops,
                    "unit": "TFLOP/s", "frac": round(achieved / tflops, 4),
                    "peak_source": f"{peak_src} dense bf16 (burst)", "traffic": profiled_traffic(spec.name)}
        extra = {"tokens_per_s": round(step_tokens / (step_ms * 1e-3), 1),
                 "kv_gbs": round(kv_gbs, 1),
                 "frac_of_sustained_bf16": round(achieved / tflops_sus, 4) if tflops_sus else None}

    cpu = None
    if dist.rank == 0 and n == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec, step, args.cpu_seconds, args.cpu_seconds_1thread)

    if dist.rank == 0:
        cfg = workload_config(spec, step, n)
        line = {"metric": metric, "value": round(value, 2), "unit": unit, "n_gpus": n, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
                **extra, **bench.details(), "roofline": roof, "cpu_baseline": cpu,
                "e2e": ({"value": round(step_work / (1e9 if spec.kind == 'decode' else 1e12) / (e2e * 1e-3), 2),
                         "unit": unit, "ms_per_step": round(e2e, 4), "h2d_bytes_per_step": h2d_bytes,
                         "d2h_bytes_per_step": d2h_bytes} if e2e else None),
                "gpu_launches": n * bench.launches_per_step * args.steps, "clocks": clocks,
                "launch": "cuda graph per step" if use_graph else "eager",
                "kernel_source_digest": source_digest()}
        print(json.dumps(line), flush=True)
    del graphs
    dist.close()


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
