"""bench.py's command-line contract, checked on the CPU: the reference arm's
JSON line, rank handling, and that the CUDA arm fails loudly without a GPU
(it never falls back to the CPU)."""

import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"]


def _run(args, **env):
    e = dict(os.environ)
    e.update(env)
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=e, capture_output=True, text=True,
                          timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "1", "--workload", "tiny_l1024"],
             BB_REF_STEP_SECONDS="0.2", RANK="0", WORLD_SIZE="1")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for k in KEYS:
        assert k in line, k
    assert line["impl"] == "reference" and line["warmup"] >= 3 and line["steps"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True and line["unit"] == "TFLOP/s"
    assert line["config"]["workload"] == "tiny_l1024"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"] and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1


def test_reference_arm_other_ranks_print_nothing():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "tiny_l1024"],
             BB_REF_STEP_SECONDS="0.2", RANK="1", WORLD_SIZE="2")
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_cuda_arm_fails_loudly_without_a_gpu():
    r = _run(["--steps", "1", "--warmup", "3", "--workload", "tiny_l1024", "--no-cpu-baseline"], RANK="0",
             WORLD_SIZE="1")
    assert r.returncode != 0
    assert '"value"' not in r.stdout
