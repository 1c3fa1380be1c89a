"""The benchmark's reference arm (the float64 oracle on host cores) prints
one JSON line with the keys the benchmark contract asks for, and refuses
fewer than three warm-up steps. CPU only: the reference arm never touches a
GPU, and our own arm refuses to run without one."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=timeout, cwd=ROOT)


def test_reference_arm_prints_the_contract_line():
    # the batched workload's bounded sample: one sequence, about 2 GB of
    # float64 weights on the host
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "batched_decode_b64_k16"


def test_reference_arm_of_the_stack_says_unavailable():
    r = _bench("--impl", "reference", "--workload", "qwen3_8b_stack_b64_k16", "--steps", "1",
               "--warmup", "3")
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and "unavailable" in line


def test_fewer_than_three_warmups_are_refused():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "2")
    assert r.returncode != 0


def test_our_arm_needs_a_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    r = _bench("--steps", "1", "--warmup", "3", "--no-cpu-baseline")
    assert r.returncode != 0 and "CUDA device" in (r.stderr + r.stdout)
