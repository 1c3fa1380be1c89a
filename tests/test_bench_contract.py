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


def test_sweep_covers_the_verifier_sweep_grid():
    """Every (B, K, dtype) of the verifier sweep at sigma = 1, plus the
    high- and low-acceptance noise levels at B = 64, K = 16, bf16."""
    import bench
    pts = bench.sweep_points()
    grid = {(B, K, dt) for B in (1, 8, 32, 64, 128, 256) for K in (4, 8, 16, 32)
            for dt in ("bf16", "f32")}
    assert {(B, K, dt) for B, K, dt, s in pts if s == 1.0} == grid
    assert {s for B, K, dt, s in pts if (B, K, dt) == (64, 16, "bf16")} == {0.25, 1.0, 4.0}
    # logits of 2K+1 rows per sequence, then the drafts and the outputs
    assert bench.verify_algorithmic_bytes(2, 3, 10, 2) == 2 * 7 * 10 * 2 + 2 * 3 * 4 + 2 * 5 * 4


def test_sweep_reference_arm_says_why_it_is_unavailable(capsys):
    import bench
    import sys
    argv = sys.argv
    sys.argv = ["bench.py", "--impl", "reference", "--workload", "verifier_sweep"]
    try:
        assert bench.main() == 0
    finally:
        sys.argv = argv
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and "unavailable" in line
