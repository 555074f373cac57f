"""Host-side pieces of bench.py that need no GPU: the kernel-source digest that
keys the measured DRAM traffic, and the JSON `config` both arms print."""
import bench
from paged_kv_attention_mg_b200 import workload as wl


def test_digest_ignores_comments_and_layout_but_not_code():
    a = 'int f(int x) { return x + 1; } // add one\n/* note */ const char *s = "// kept";\n'
    b = 'int f(int x)\n{\n    return x + 1;  // a different comment\n}\nconst char *s = "// kept";\n'
    c = 'int f(int x) { return x + 2; }\nconst char *s = "// kept";\n'
    d = 'int f(int x) { return x + 1; }\nconst char *s = "// changed";\n'
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)   # code change
    assert bench._code_only(a) != bench._code_only(d)   # string literals are code


def test_digest_is_stable_and_hex():
    d = bench.source_digest()
    assert d == bench.source_digest() and len(d) == 16 and int(d, 16) >= 0


def test_both_arms_share_the_workload_config():
    for name in ("qwen3_0.6b_decode_28l", "chunked_prefill_extend"):
        spec = wl.BY_NAME[name]
        step = wl.make_step(spec)
        cfg = bench.workload_config(spec, step, 1)
        assert cfg["workload"] == name and cfg["parallelism"] == "single GPU"
        assert cfg["batch"] == spec.batch and cfg["q_heads"] == spec.num_q_heads
        assert bench.workload_config(spec, step, 4)["parallelism"].startswith("dp4")


def test_oracle_sampler_generates_inputs_once_and_fills_its_time_bound():
    import oracle
    oracle.build()
    spec = wl.BY_NAME["tiny_decode"]
    step = wl.make_step(spec)
    sampler = bench.OracleSampler(spec, step, threads=1, max_layers=2)
    for _ in range(3):
        work, secs, sample, unit = sampler.sample(0.05)
        assert unit == "GB/s" and secs >= 0.05 and work > 0
        assert work % bench.rf.decode_bytes(step.seq_len.tolist(), spec.num_q_heads, spec.num_kv_heads,
                                            spec.head_dim) == 0
    assert len(sampler._layers) == min(2, spec.num_layers)   # held across samples, never regenerated
    ext = wl.custom_spec("extend", [0, 5], [9, 12], 4, 2, 64, seed=3)
    es = bench.OracleSampler(ext, wl.make_step(ext), threads=1)
    work, secs, sample, unit = es.sample(0.0)
    assert unit == "TFLOP/s" and work > 0 and "1 requests" in sample and len(es._layers) == 1


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun the oracle arm is rank 0's alone: other ranks print nothing and exit."""
    import argparse
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload="tiny_decode", steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_a_small_workload(monkeypatch, capsys):
    import argparse
    import json
    monkeypatch.setenv("RANK", "0")
    args = argparse.Namespace(workload="tiny_decode", steps=2, warmup=1, gpus=1)
    monkeypatch.setattr(bench, "cpu_threads", lambda: 1)
    bench.run_reference(args)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["config"]["workload"] == "tiny_decode" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["steps"] == 2 and line["warmup"] == 1


def test_committed_bench_lines_follow_the_contract():
    """Every bench line committed under profiles/ carries the keys the bench
    contract asks for, and its traffic figure is the one profiles/traffic.json
    holds for its workload at the same kernel-source digest (never a figure
    taken on other kernels)."""
    import glob
    import json
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    traffic = json.load(open(os.path.join(root, "profiles", "traffic.json")))
    paths = sorted(glob.glob(os.path.join(root, "profiles", "bench_*.json")))
    assert paths
    for path in paths:
        line = json.loads(open(path).read())
        for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                    "scaling", "vs_baseline", "dtype", "data", "config", "e2e", "cpu_baseline"):
            assert key in line, (path, key)
        assert line["warmup"] >= 3 and line["steps"] >= 1, path
        e2e = line["e2e"]
        assert {"value", "unit"} <= set(e2e), path
        cpu = line["cpu_baseline"]
        assert {"value", "unit", "cores", "kind", "sample"} <= set(cpu) and cpu["kind"] == "oracle", path
        if line.get("impl") == "reference":
            continue
        assert "workload" in line["config"], path
        assert line["gpu_launches"] > 0, path
        clocks = line["clocks"]
        assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(clocks), path
        assert not {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"} & set(clocks["reasons"]), path
        assert {"h2d_bytes_per_step", "d2h_bytes_per_step"} <= set(e2e), path
        roof = line["roofline"]
        assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(roof), path
        assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-3, path
        if roof["traffic"] is not None:
            key = line["config"]["workload"] + (":plain" if "plain" in os.path.basename(path) else "")
            assert traffic[key]["source_digest"] == line["kernel_source_digest"], path
            assert traffic[key]["dram_bytes_per_launch"] == roof["traffic"], path
