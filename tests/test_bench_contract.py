"""bench.py's reference arm (the oracle, timed on the host cores) prints the
JSON line the driver parses, and needs no GPU; under several ranks only rank
0 prints it."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _run(extra_env, *args):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", **extra_env)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=900, env=env)


def test_reference_arm_prints_the_contract_line():
    out = _run({}, "--steps", "2", "--warmup", "3", "--ref-tokens", "4", "--layer", "tiny")
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1
    assert d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert "workload" in d["config"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    # the reference line describes the same workload as the GPU arm's line
    assert d["config"] == bench.bench_config("tiny", 16, 1)
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    out = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--steps", "1", "--ref-tokens", "2",
               "--layer", "tiny")
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""
