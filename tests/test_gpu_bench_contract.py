"""The benchmark's JSON line (one GPU, a small workload): every key the
measurement contract names is there and consistent with the run."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    cmd = [sys.executable, "bench.py", "--steps", "4", "--warmup", "3", "--no-extras", *args]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_line_carries_the_contract_keys():
    d = _run("--workload", "tiny")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
              "cpu_baseline"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["config"]["workload"].startswith("tiny layer")
    roof = d["roofline"]
    assert roof["bound"] in ("tensor", "hbm", "alu") and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) <= 1e-9 * max(1.0, roof["frac"])
    assert len(roof["peak_per_gemm"]) == roof["launches_per_step"] == 4
    cold = d["kernels_cold_l2"]
    assert {"dispatch", "combine", "edge_aggregate"} <= set(cold) and all(v["ms"] > 0 for v in cold.values())
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    # this library's kernels per step: route 4, edge aggregation 1, dispatch 1,
    # MLP 2 + 2, combine 1 + 1, weighted dispatch 1 (the tiny layer's 128 rows
    # per expert stay below the FP16 tensor path's threshold)
    assert d["gpu_launches"] == 13 * d["steps"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"] and d["clocks"]["samples_in_timed_region"] >= 1


def test_reference_arm_line():
    d = _run("--workload", "tiny", "--impl", "reference", "--ref-seconds", "1")
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
