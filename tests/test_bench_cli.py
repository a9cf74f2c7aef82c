"""bench.py's command line on a host without a GPU: argument checks and the
reference arm's lines for the workloads that have no reference."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=300, env=env)


def test_warmup_below_three_is_rejected():
    p = _run("--warmup", "2")
    assert p.returncode == 2 and "--warmup must be >= 3" in p.stderr


@pytest.mark.parametrize("config", ["act-codec", "swiglu-fp8", "rmsnorm-fp8"])
def test_reference_arm_of_layer_and_codec_workloads_is_unavailable(config):
    p = _run("--impl", "reference", "--config", config)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and "unavailable" in rec


def test_reference_arm_single_process_line():
    p = _run("--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-sample", "4096")
    assert p.returncode == 0, p.stderr[-2000:]
    rec = json.loads([l for l in p.stdout.splitlines() if l.startswith("{")][0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "cpu_baseline", "e2e", "config"):
        assert key in rec, key
    assert rec["n_gpus"] == 1 and rec["cpu_baseline"]["cores"] == len(os.sched_getaffinity(0))
    assert rec["config"]["sample_elements"] == 8 * 4096 + 2 * 4096   # 10 tensors of the 7B slice
