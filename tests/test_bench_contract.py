"""The benchmark's command-line contract, on the CPU.

The reference arm times the oracle on the host cores and must print one JSON
line with the contract's keys; the GPU arm must refuse to run (exit non-zero)
when there is no CUDA device rather than fall back to the CPU.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(*args, timeout=600):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    p = run("--impl", "reference", "--steps", "1", "--warmup", "3",
            "--reference-fraction", "0.002")
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert "workload" in d["config"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_bench_rejects_fewer_than_three_warmup_steps():
    p = run("--impl", "reference", "--steps", "1", "--warmup", "2", timeout=120)
    assert p.returncode != 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU refusal")
def test_gpu_arm_fails_loudly_without_a_device():
    p = run("--steps", "1", "--warmup", "3", "--no-cpu-baseline", "--no-e2e", timeout=300)
    assert p.returncode != 0
    d = json.loads(p.stdout.strip().splitlines()[-1])
    assert "error" in d and "value" not in d
