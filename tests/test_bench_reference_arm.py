"""The bench's reference arm (the fp64 oracle on the host cores) runs on the
CPU and prints one JSON line in the contract's format."""

import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_a_contract_line():
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
                        "--warmup", "3", "--cpu-budget", "0.5"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    wall_ms = (time.perf_counter() - t0) * 1e3
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] >= 3
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("tiny")
    # ms_per_step is a time the run really contains; the extrapolated layer
    # time is reported under its own key
    assert 0 < d["ms_per_step"] and d["steps"] * d["ms_per_step"] < wall_ms
    assert d["extrapolated_layer_ms"] > 0
