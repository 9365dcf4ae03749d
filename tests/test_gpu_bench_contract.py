"""bench.py's JSON line carries the measurement keys, on a short run.

The line is what a benchmark driver reads: throughput of whole steps, the
roofline of the dominant kernel (frac = achieved / peak), the oracle timed on
the host, the end-to-end figure through host buffers, the launch count and
the SM clocks seen during the timed region."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_has_the_measurement_keys():
    steps = 40
    cmd = [sys.executable, "bench.py", "--steps", str(steps), "--warmup", "3", "--isolated-steps", "20",
           "--e2e-steps", "10", "--fp32-steps", "10", "--cpu-seconds", "1", "--no-graph"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches", "clocks"):
        assert key in d, key
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, steps, 3)
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["gpu_launches"] == 2 * steps
    assert d["config"]["workload"].startswith("gdn")
    rf = d["roofline"]
    assert rf["bound"] in ("alu", "hbm", "tensor") and rf["peak"] > 0 and rf["achieved"] > 0
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) <= 1e-9 * rf["frac"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]
