"""bench.py's host-side contract on CPU: the reference arm (the fp64 oracle on sampled rows)
prints one JSON line with the required keys, and the helpers that turn measurements into the
reported figures (whole-job throughput, attention DRAM traffic) behave as documented."""
import json
import os
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]


def test_reference_arm_prints_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    sys.path.insert(0, str(ROOT))
    import bench
    assert j["metric"] == bench.METRIC and j["impl"] == "reference"
    for key in ("value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["value"] > 0 and j["unit"] == "TFLOP/s" and j["higher_is_better"] is True
    assert j["config"]["workload"] == "fp8-128k"
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["cpu_baseline"]["cores"] >= 1 and j["cpu_baseline"]["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_throughput_and_traffic_helpers(monkeypatch):
    sys.path.insert(0, str(ROOT))
    import bench
    # weak scaling: every rank runs the full problem; 1e12 FLOP in 1 s per rank
    assert bench.whole_job_tflops(1e12, 1, 1000.0) == pytest.approx(1.0)
    assert bench.whole_job_tflops(1e12, 8, 1000.0) == pytest.approx(8.0)
    # DRAM traffic of the default kernel is linear in tokens; other kernels / shapes report null
    monkeypatch.delenv("BSA_ATTN_VARIANT", raising=False)
    t1 = bench.attn_traffic(True, 1, 32768, 64, 8, 128)
    assert t1 == pytest.approx(358.912512e6 + 485.153280e6)
    assert bench.attn_traffic(True, 1, 131072, 64, 8, 128) == pytest.approx(4 * t1)
    assert bench.attn_traffic(True, 2, 32768, 64, 8, 128) == pytest.approx(2 * t1)
    assert bench.attn_traffic(False, 1, 32768, 64, 8, 128) is None
    monkeypatch.setenv("BSA_ATTN_VARIANT", "serial")
    assert bench.attn_traffic(True, 1, 32768, 64, 8, 128) is None


def test_reference_arm_other_ranks_exit_without_work():
    """Under torchrun only rank 0 runs and prints the reference line; the others exit 0 at once."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]
