"""bench.py's per-workload line and roofline arithmetic, on made-up timings (no GPU)."""
import importlib.util
import os

import numpy as np

from mla_decode_attention_12_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_workload_line_fields_and_roofline():
    b = _bench()
    p = W.make_problem([1024, 2048], s_q=1, h_q=128, seed=5, name="compute")
    rng = np.random.default_rng(0)
    t = np.stack([rng.uniform(0.10, 0.12, 50), np.full(50, 0.008), np.full(50, 0.1), np.full(50, 0.014)], 1)
    peaks = {"hbm_gbs": 6540.8, "bf16_tflops": 1656.2, "bf16_tflops_sustained": 1371.4}
    line = b.workload_line(p, t, peaks, "measured")
    assert line["us_per_call_p10"] <= line["us_per_call_median"] <= line["us_per_call_p90"]
    assert abs(line["us_splitkv"] - 100.0) < 1e-6
    rf = line["roofline"]
    # achieved = algorithmic bytes (or flops) / the split-KV time; frac = achieved / peak
    if rf["bound"] == "hbm":
        assert abs(rf["achieved"] - p.io_bytes() / 100e-6 / 1e9) < 0.01
    else:
        assert abs(rf["achieved"] - p.flops() / 100e-6 / 1e12) < 0.01
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-3
    assert line["kv_gbs"] > 0 and line["tflops"] > 0


def test_code_hash_ignores_comments_only():
    b = _bench()
    code = 'int f(int a) { return a + 1; } // one\n/* two */ const char* s = "x // y";'
    assert b._code_tokens(code) == b._code_tokens(code.replace("// one", "// changed").replace("two", "2"))
    assert b._code_tokens(code) != b._code_tokens(code.replace("a + 1", "a + 2"))
    assert b._code_tokens(code) != b._code_tokens(code.replace('"x // y"', '"x // z"'))


def test_reference_arm_prints_the_gpu_arms_config(capsys, monkeypatch):
    # The two arms of one workload carry identical config objects, so their lines compare
    # directly.  The reference arm runs the oracle on a tiny bounded sample here.
    import json
    import sys

    b = _bench()
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
                                      "--warmup", "0"])
    monkeypatch.setenv("WORLD_SIZE", "1")
    b.main()
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == b.workload_config(W.make_workload("tiny"), 1)
