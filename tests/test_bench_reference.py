"""bench.py --impl reference (the CPU oracle on a bounded sample) prints one
JSON line with the contract's keys, on the same config as the GPU arm."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def _check_contract(line):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


@pytest.mark.parametrize("workload", ["decode", "split"])
def test_reference_arm_kv_workloads(workload):
    import bench

    line = _run("--workload", workload, "--steps", "2", "--warmup", "1")
    _check_contract(line)
    bench.set_workload(workload)
    assert line["config"] == bench.kv_config(1)
    assert line["unit"] == "keys/s" and line["scaling"] == "weak"


def test_reference_arm_search():
    import bench

    line = _run("--workload", "search", "--rows", "30000", "--queries", "200", "--steps", "2", "--warmup", "1")
    _check_contract(line)
    assert line["config"] == bench.search_config(30000, 200, 200, 10, 1)
    assert line["metric"] == bench.SEARCH_METRIC and line["unit"] == "queries/s" and line["scaling"] == "strong"
