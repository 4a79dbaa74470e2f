"""The reference arm of bench.py (the oracle on host cores) prints one JSON
line with the contract's keys, for the attention, FFN and decode workloads.
Runs on CPU: the reference arm touches no GPU."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup",
        "ms_per_step", "higher_is_better", "scaling", "vs_baseline", "dtype",
        "data", "config", "cpu_baseline", "e2e"}


def _run(workload, extra=()):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--workload",
         workload, "--steps", "1", "--warmup", "0", "--ref-budget", "0.05",
         *extra],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("workload,unit", [("packed128k", "TFLOP/s"),
                                           ("text32k", "TFLOP/s"),
                                           ("mlp8k", "TFLOP/s"),
                                           ("decode1m", "GB/s")])
def test_reference_line(workload, unit):
    d = _run(workload)
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["unit"] == unit
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["warmup"] >= 3 and d["steps"] == 1
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"] == workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"]
    assert cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": unit,
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_other_ranks_print_nothing():
    env_rank = {"RANK": "1", "WORLD_SIZE": "2"}
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", **env_rank)
    r = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--workload",
         "decode1m", "--steps", "1", "--warmup", "0", "--ref-budget", "0.05"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and not r.stdout.strip()


def test_default_workload_is_packed_128k():
    # the 128K packed configuration is what the forward / backward targets
    # are stated on: the bench runs it when no workload is named
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
         "--warmup", "0", "--ref-budget", "0.05"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][0])
    assert d["config"]["workload"] == "packed128k"
