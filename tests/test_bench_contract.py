"""bench.py's reference arm (the fp64 oracle timed on the host cores) keeps
the benchmark's JSON contract: one line with the metric, unit, config and
timing keys of the GPU arm, plus cpu_baseline and e2e.  It runs on a CPU
in seconds, so it is checked end to end here; the GPU arm prints the same
metric and config (bench.METRIC, bench.workload_config)."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600, check=True)
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, out.stdout
    r = json.loads(lines[0])
    assert r["impl"] == "reference"
    assert r["metric"] == bench.METRIC and r["unit"] == "TFLOP/s"
    assert (r["n_gpus"], r["steps"], r["warmup"]) == (1, 1, 0)
    assert r["value"] > 0 and r["ms_per_step"] > 0
    assert r["higher_is_better"] is True and r["scaling"] == "weak" and r["vs_baseline"] is None
    assert r["dtype"] == "f64" and r["data"] == "synthetic"
    assert r["config"] == json.loads(json.dumps(bench.workload_config(1)))   # the GPU arm's config
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["unit"] == r["unit"]
    assert cb["cores"] >= 1 and cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": r["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
