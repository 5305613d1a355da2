"""The reference arm of the benchmark (the oracle on the host cores) prints one
JSON line with the contract's keys and the same metric, unit and workload as
the CUDA arm (CPU only; a few seconds)."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_json_line():
    d = _run("--impl", "reference", "--steps", "1", "--warmup", "0")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["higher_is_better"] is True
    assert d["config"]["workload"] == "llama3_8b_prefill"
    # the same metric and unit as the CUDA arm
    assert d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    """Under a multi-rank launch only rank 0 runs the oracle and prints."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert not [l for l in out.stdout.splitlines() if l.startswith("{")]


def test_gpus_must_match_the_launched_world_size():
    """Under a distributed launch --gpus N must equal WORLD_SIZE, so that the
    line's n_gpus is the number of ranks that did the work (both arms)."""
    env = dict(os.environ, RANK="0", LOCAL_RANK="0", WORLD_SIZE="2")
    for impl in ("reference", "ours"):
        out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", impl, "--gpus", "4",
                              "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                             timeout=300)
        assert out.returncode == 2, (impl, out.returncode, out.stderr[-2000:])
        assert "WORLD_SIZE=2" in out.stderr
        assert not [l for l in out.stdout.splitlines() if l.startswith("{")]
