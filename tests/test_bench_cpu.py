"""bench.py on the CPU: the reference arm's JSON line (the oracle timed on the
host) and the GPU arm's refusal to run without a CUDA device."""
import json
import os
import subprocess
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          cwd=ROOT, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = run_bench("--impl", "reference", "--workload", "sweep-quick", "--steps", "1", "--warmup", "3",
                  "--ref-rows", "2")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["ms_per_step"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_rejects_too_few_warmups():
    r = run_bench("--impl", "reference", "--workload", "sweep-quick", "--steps", "1", "--warmup", "1")
    assert r.returncode != 0


def test_gpu_arm_refuses_without_cuda():
    if torch.cuda.is_available():
        return  # only meaningful on a machine without a GPU
    r = run_bench("--workload", "sweep-quick", "--steps", "1", "--warmup", "3")
    assert r.returncode != 0
    assert "CUDA" in (r.stderr + r.stdout)
