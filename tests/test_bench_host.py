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
