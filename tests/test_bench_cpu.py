"""bench.py contract checks that need no GPU: the reference arm (the oracle on
the host cores) prints one JSON line with the contract's keys, and our arm
refuses to run without a CUDA device instead of falling back to the CPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=240):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_the_contract_line():
    r = _run("--impl", "reference", "--workload", "smoke-256", "--steps", "2", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] >= 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "smoke-256"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert cb["unit"] == d["unit"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_default_workload_states_host_cores():
    """The default workload (the training-batch forward) on the reference arm:
    the oracle on a token sample, the threads it used and the host's cores."""
    r = _run("--impl", "reference", "--steps", "2", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")][0])
    assert d["config"]["workload"] == "train-fwd-1.3b" and d["config"]["M"] == 524288
    cb = d["cpu_baseline"]
    assert cb["host_cores"] >= 1 and cb["threads"] >= 1 and cb["cores"] == cb["threads"]
    assert "extrapolated" in cb["sample"]


@pytest.mark.parametrize("workload", ["smoke-256", "decode-2.7b-m1", "train-fwd-1.3b"])
def test_our_arm_fails_loudly_without_a_device(workload):
    r = _run("--workload", workload, "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    assert r.returncode != 0
    assert "CUDA device" in (r.stderr + r.stdout)
    assert not any(ln.strip().startswith("{") for ln in r.stdout.splitlines())
