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
