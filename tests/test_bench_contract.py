"""The benchmark's JSON line, checked on CPU: the reference arm (the oracle on the host cores)
on the small prefill geometry prints every key of the contract, with the same `config` object
the product arm prints for that workload."""
import argparse
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--small", "--steps", "1",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "e2e", "cpu_baseline"):
        assert k in j, k
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC and j["unit"] == "queries/s"
    assert j["higher_is_better"] is True and j["steps"] == 1 and j["warmup"] == 3 and j["value"] > 0
    assert set(j["e2e"]) == {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert j["e2e"]["value"] == j["value"] and j["e2e"]["h2d_bytes_per_step"] == 0
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"] and cb["sample"]
    assert j["config"] == bench.prefill_config(bench.bench_config(argparse.Namespace(small=True)), 1)
