"""bench.py's reference arm (the fp64 oracle timed on the host cores) runs
without a GPU and prints one JSON line with the keys the bench contract asks
for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
         "--warmup", "3", "--workload", "0", "--cpu-seconds", "0.2"],
        capture_output=True, text=True, timeout=600, cwd=ROOT, check=True).stdout
    lines = [l for l in out.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "full_b1_h2_s256_d64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_names_a_grouped_query_config():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
         "--warmup", "3", "--workload", "0", "--cpu-seconds", "0.2", "--kv-heads", "1"],
        capture_output=True, text=True, timeout=600, cwd=ROOT, check=True).stdout
    d = json.loads([l for l in out.splitlines() if l.strip().startswith("{")][-1])
    assert d["config"]["workload"] == "full_b1_h2_s256_d64_kv1"
    assert d["config"]["H"] == 2 and d["config"]["H_kv"] == 1
    assert d["value"] > 0
