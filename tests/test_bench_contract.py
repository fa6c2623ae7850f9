"""The benchmark's output contract, checked on the CPU: `bench.py --impl reference` (the
oracle on the host cores, no GPU) prints one JSON line with the metric, unit and keys the
benchmark promises, and under torchrun only rank 0 prints it (the other ranks exit 0 without
work). The training arm's own line needs a GPU; its key set is the same contract."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None, timeout=240):
    env = dict(os.environ, PYTHONPATH=ROOT, **(env_extra or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


@pytest.mark.slow
def test_reference_arm_prints_one_json_line():
    r = _run(["--impl", "reference", "--workload", "tiny_2of4", "--steps", "2", "--warmup", "3",
              "--ref-step-seconds", "0.2"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["metric"] and d["unit"] == "blocks/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny_2of4"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_on_other_ranks():
    r = _run(["--impl", "reference", "--workload", "tiny_2of4", "--steps", "1"], {"RANK": "1", "WORLD_SIZE": "2"},
             timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_warmup_is_raised_to_three():
    r = _run(["--impl", "reference", "--workload", "tiny_2of4", "--steps", "1", "--warmup", "1",
              "--ref-step-seconds", "0.1"], timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert json.loads(r.stdout.strip().splitlines()[-1])["warmup"] == 3


def test_serve_nm_is_only_for_the_serving_mode():
    """--serve-nm repacks a workload for the serving benchmark only; the training step keeps
    the workload's own pattern (its 4:8 state would not fit for the full stack)."""
    r = _run(["--serve-nm", "4:8", "--workload", "tiny_2of4", "--steps", "1"], timeout=120)
    assert r.returncode != 0
    assert "--serve-nm applies to --mode sparse_linear" in r.stderr
