"""The bounds-checked build: every global, shared and tensor-memory index of the decode,
quantize and multi-token kernels compared with its extent (nvcc -DISOQ_CHECK_BOUNDS).

A child process loads libisoq_checked.so (ISOQ_CHECK_BOUNDS=1) and runs the 1024-token
workload, the 32k-token d = 256 workload, a ragged paged batch with appends, both
multi-token kernels, the 2- and 4-bit formats, and the RoPE-fused and layer-batched
appends; every case must end with status 0 and parity green.  The self-test
shows the check is live there (ISOQ_ST_BOUNDS set for an index equal to its extent) and
compiled out of the normal library (status clear)."""
import json
import os
import subprocess
import sys

import pytest
import torch

import rotated_bit_kv_isoquant_b200 as iq

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED_LIB = os.path.join(ROOT, "rotated_bit_kv_isoquant_b200", "libisoq_checked.so")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _build_checked():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_isoq_build", os.path.join(ROOT, "rotated_bit_kv_isoquant_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b.build(checked=True)


def test_normal_build_compiles_the_check_out():
    assert not iq.CHECKED
    assert iq.isoq_selftest_bounds() == 0


def test_checked_build_runs_clean():
    assert _build_checked() == CHECKED_LIB
    env = dict(os.environ, ISOQ_CHECK_BOUNDS="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_checked_cases.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=1800)
    sys.stdout.write(p.stdout)
    recs = {}
    for line in p.stdout.splitlines():
        if line.startswith("{"):
            r = json.loads(line)
            recs[r["case"]] = r
    assert p.returncode == 0, p.stdout[-4000:] + p.stderr[-4000:]
    assert recs["selftest"]["status"] == iq.ISOQ_ST_BOUNDS
    for name in ("cfg1", "cfg3", "ragged", "multi_mq", "multi_tc", "formats", "rope_layers"):
        assert recs[name]["ok"] and recs[name]["status"] == 0, recs[name]
