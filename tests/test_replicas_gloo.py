"""The data-parallel (replica) path of bench.py on CPU ranks: world size 2
over gloo.

One decode step shards by batch: every rank verifies its own B sequences
and runs its own dual-path projections, with no exchange on the data path.
What the ranks share is the bookkeeping around the timed region, which this
test runs on gloo: the max over ranks of the step time, the whole-job rate
computed from it, and the per-replica seeds (each replica must draw its own
inputs and its own acceptance / resampling uniforms).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

WORLD = 2
ROWS_PER_STEP = 64 * 16
LOCAL_MS = (3.25, 5.5)  # one slow rank


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, port: int, out_dir: str) -> None:
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=WORLD,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from lossless_decoding_b200.inputs import verify_inputs
        from oracle import uno_oracle

        cpu = torch.device("cpu")
        ms = bench.max_over_ranks(LOCAL_MS[rank], WORLD, cpu)
        rate = bench.whole_job_rate(ROWS_PER_STEP, WORLD, ms)
        input_seed, key = bench.replica_seeds(rank)
        v = verify_inputs(2, 4, 64, dtype="f32", seed=input_seed, device=cpu)
        u_acc, u_smp = uno_oracle.uniforms_for_block(2, 4, key, step=7)
        gathered = [None] * WORLD
        torch.distributed.all_gather_object(
            gathered, (ms, rate, input_seed, key, v.p_logits.numpy().tolist(),
                       u_acc.tolist(), u_smp.tolist()))
        if rank == 0:
            torch.save(gathered, os.path.join(out_dir, "gathered.pt"))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


@pytest.fixture(scope="module")
def gathered(tmp_path_factory):
    out = tmp_path_factory.mktemp("replicas")
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, str(out))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    codes = [p.exitcode for p in procs]
    assert codes == [0] * WORLD, f"gloo ranks exited with {codes}"
    return torch.load(out / "gathered.pt", weights_only=False)


def test_step_time_is_max_over_ranks(gathered):
    for ms, *_ in gathered:
        assert ms == max(LOCAL_MS)


def test_whole_job_rate_counts_every_rank(gathered):
    for _, rate, *_ in gathered:
        assert rate == pytest.approx(WORLD * ROWS_PER_STEP / (max(LOCAL_MS) / 1e3), rel=1e-12)


def test_replicas_draw_their_own_inputs_and_uniforms(gathered):
    (_, _, s0, k0, p0, ua0, us0), (_, _, s1, k1, p1, ua1, us1) = gathered
    assert s0 != s1 and k0 != k1
    assert not np.array_equal(np.asarray(p0), np.asarray(p1))
    assert not np.array_equal(np.asarray(ua0), np.asarray(ua1))
    assert not np.array_equal(np.asarray(us0), np.asarray(us1))


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(2.5, 1, torch.device("cpu")) == 2.5
    assert bench.whole_job_rate(100, 1, 10.0) == pytest.approx(1e4)
