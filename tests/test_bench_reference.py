"""The reference arm of bench.py (the C oracle on the host cores) runs without a GPU and prints
the contract's JSON line."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "1", "--ref-seconds", "3"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("c5")


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_algorithmic_bytes_and_launch_counts():
    """The bytes each timed op must move, counted from the formats, and the nested quantize's
    launch count (codes, one per offset-tree level above 2048 values, the compression)."""
    b = _bench_module()
    n = 16384 * 16384
    nb = n // 32
    assert b.op_bytes("quantize", n, 3) == 2 * n + nb * 3 * 4 + nb * 4 == 671088640
    assert b.op_bytes("dequantize", n, 5) == nb * 5 * 4 + nb * 4 + 2 * n == 738197504
    assert b.op_bytes("nested", n) == n // 2 + n // 64 + n // 64 // 256 * 4 + 2 * n
    for bs in (64, 32):
        nbo = n // bs
        assert b.op_bytes("quantize_4bit", n, bs) == 2 * n + n // 2 + nbo * 4
        assert b.op_bytes("quantize_nested", n, bs) == 2 * n + n // 2 + nbo + nbo // 256 * 4 + 4
    assert b.nested_quant_launches(n, 64) == 3                 # 4,194,304 blocks: one tree level
    assert b.nested_quant_launches(n // 2 + 32 * 5000, 32) == 4  # above 2048 * 2048 blocks: two
    assert b.nested_quant_launches(2048 * 64, 64) == 2          # the root alone, inside the compression
    names = [o[0] for o in b.workload_ops("quantize_nested_nf4_bs32,quantize_4bit_nf4_bs64,dequantize_k4")]
    assert names == ["dequantize_k4", "quantize_4bit_nf4_bs64", "quantize_nested_nf4_bs32"]


def test_both_arms_name_the_same_config():
    bench = _bench_module()
    ops = bench.ALL_OPS
    assert bench.workload_desc(bench.N_C5, ops, 1) == bench.workload_desc(bench.N_C5, list(ops), 1)
    assert bench.workload_desc(bench.N_C5, ops, 1)["parallelism"] == "single"
    assert bench.workload_desc(bench.N_C5, ops, 4)["parallelism"] == "replicas4"


def test_gpus_must_match_the_ranks_started():
    import subprocess
    import sys
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode != 0 and "WORLD_SIZE=1" in r.stderr
