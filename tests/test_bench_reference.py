"""The reference arm of bench.py: the oracle timed on the host cores, one
bounded sample of the workload per step, on the same metric and config keys as
the GPU arm. Runs on the CPU (the 32K layer keeps it to a few seconds)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, *args):
    env = dict(os.environ, **(extra_env or {}))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        *args], capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_line_keeps_the_contract():
    lines = _run(None, "--config", "c1", "--steps", "2", "--warmup", "1")
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["unit"] == "ms/layer" and d["higher_is_better"] is False
    assert d["value"] > 0 and d["ms_per_step"] == d["value"]
    assert d["config"]["L"] == 32768 and d["config"]["S"] == 8
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "query blocks" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "ms/layer", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_other_ranks_do_nothing():
    """Under torchrun only rank 0 runs the oracle and prints; the others exit 0."""
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}, "--config", "c1", "--steps", "1") == []
