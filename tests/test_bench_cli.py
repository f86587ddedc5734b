"""bench.py's command-line contract, on the CPU.

- The reference arm (`--impl reference`: the oracle on the host cores) prints
  one JSON line with the metric, unit, direction, a cpu_baseline describing
  the run and an e2e block with no host-device bytes; ranks other than 0
  print nothing and exit 0.
- The GPU arm has no CPU fallback: without a CUDA device it exits non-zero.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SMALL = ["--shape", "4,256,8,2,128,fp8", "--steps", "2", "--warmup", "1"]


def _run(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=e, capture_output=True, text=True,
                          timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run(["--impl", "reference", *SMALL])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert (d["steps"], d["warmup"], d["n_gpus"]) == (2, 1, 1)
    assert d["config"]["workload"] == "custom_T4_H256_E8_k2_I128_fp8"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", *SMALL], env={"RANK": "1"})
    assert r.returncode == 0 and not r.stdout.strip()


def test_gpu_arm_has_no_cpu_fallback():
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present: the GPU arm runs")
    r = _run(SMALL)
    assert r.returncode != 0
    assert not r.stdout.strip()
