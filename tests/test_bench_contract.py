"""bench.py's command line and the JSON line of its reference arm (CPU: the float64 oracle).

The GPU arm prints the same keys plus roofline, clocks and gpu_launches; it needs a device and
is exercised by the bench runs themselves."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, env=None, timeout=600):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout,
                          env=dict(os.environ, **(env or {})))


@pytest.mark.parametrize("args,unit,workload", [
    (["--workload", "tiny_2k"], "tokens/s", "tiny_2k"),
    (["--decode"], "sequences/s", "decode_32k_b64"),
    (["--decode", "--gate", "minmax"], "sequences/s", "decode_32k_b64"),
], ids=["prefill", "decode_mean", "decode_minmax"])
def test_reference_arm_prints_one_contract_line(args, unit, workload):
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "3", *args)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["unit"] == unit and d["value"] > 0 and d["ms_per_step"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 1, 3)
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == "f64" and "synthetic" in d["data"]
    assert d["config"]["workload"] == workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == unit
    assert cb["cores"] >= 1 and isinstance(cb["sample"], str) and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == unit
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    if "--gate" in args:
        assert d["config"]["gate"] == "minmax"
    if "--decode" not in args:
        assert cb["cpu_count"] >= 1 and cb["extrapolated"] is True


def test_reference_arm_runs_on_rank_zero_only():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "3", "--decode",
             env={"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.parametrize("args", [["--warmup", "2"], ["--gate", "maxmin"]], ids=["warmup_below_3", "unknown_gate"])
def test_invalid_command_lines_are_rejected(args):
    r = _run("--impl", "reference", "--steps", "1", *args, timeout=120)
    assert r.returncode != 0 and "error" in r.stderr
