"""The benchmark's command-line contract, checked without a GPU: the reference
arm (the float64 oracle timed on host cores) prints one JSON line with the
keys and units of the GPU arm's line, the warm-up floor is enforced, and the
GPU arm fails loudly instead of falling back to anything when no GPU is
present."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _run(*args, timeout=240):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=timeout, env=env, cwd=ROOT)


def _json_lines(stdout):
    return [json.loads(s) for s in stdout.splitlines() if s.startswith("{")]


@pytest.mark.parametrize("workload", ["fwdbwd", "decode"])
def test_reference_arm_prints_one_contract_line(workload):
    r = _run("--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["data"] == "synthetic" and "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == line["value"] and cb["unit"] == line["unit"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # same metric and unit as the GPU arm of the same workload
    w = bench.WORKLOADS[workload]
    if workload == "decode":
        assert line["metric"] == bench.DECODE_METRIC and line["unit"] == "GB/s"
    else:
        assert line["metric"] == bench.kernel_names(w)[0] and line["unit"] == bench.UNIT


def test_warmup_floor_is_enforced():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "2")
    assert r.returncode != 0
    assert "--warmup must be >= 3" in r.stderr
    assert not _json_lines(r.stdout)


def test_gpu_arm_fails_loudly_without_a_gpu():
    r = _run("--steps", "3", "--warmup", "3", "--no-cpu-baseline", "--no-e2e", "--no-c3")
    assert r.returncode != 0
    assert not _json_lines(r.stdout), "a line was printed without a GPU"
