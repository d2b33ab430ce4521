"""The bench's reference arm (the oracle on the host cores) runs without a GPU and prints the
one-line JSON record the measurement contract asks for, with the same metric, unit and
direction as the CUDA arm, so that the two arms' values can be divided."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_bench", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_reference_arm_prints_the_contract_line():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    b = _load_bench()
    assert r["impl"] == "reference"
    assert r["metric"] == b.METRIC and r["unit"] == "GB/s" and r["higher_is_better"] is True
    assert r["n_gpus"] == 1 and r["steps"] == 1 and r["warmup"] == 3
    assert r["value"] > 0 and r["config"]["workload"] == "long131k_gqa8"
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1
    assert r["e2e"]["value"] == r["value"] and r["e2e"]["unit"] == r["unit"]
    assert r["e2e"]["h2d_bytes_per_step"] == 0 and r["e2e"]["d2h_bytes_per_step"] == 0
