"""Benchmark of one Psi-Spec decode step's hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload batched_decode_b64_k16|qwen3_8b_b1|qwen3_8b_stack_b64_k16
                                |verifier_sweep]

A step is one pass over the whole hot path for one batch:
  batched_decode_b64_k16 (default): B = 64 sequences x K = 16 drafted positions
      = 1024 rows; the dual-pathway linear of every projection of one
      Qwen3-8B-shaped layer (q, k, v, o, gate, up, down; rank-128 LoRA,
      alpha 256, bf16) over the 1024 rows, then the block verifier over
      64 x (2*16+1) rows of 151936 bf16 logits.
  qwen3_8b_b1: one sequence, K = 16: the dual-path LM head 4096 -> 151936 over
      the 17 rows (16 drafts + the bonus row), then the verifier on its logits
      (p = y_AR rows, q = y_draft rows).
  qwen3_8b_stack_b64_k16: the whole 8B-shaped draft-verify step: 36 layers of
      dual-path projections over 64 x 17 rows (row gate: first position AR
      only), the dual-path LM head, the on-device draft sampler, the verifier.
  verifier_sweep: the block verifier alone over every (B, K, dtype) of
      B in {1, 8, 32, 64, 128, 256}, K in {4, 8, 16, 32}, bf16 and f32,
      V = 151936, Gumbel logits with 20 tokens per row boosted by +8, draft
      noise sigma = 1 (and 0.25, 4 at B = 64, K = 16, bf16): GB/s and the
      fraction of the HBM peak per point, one step = one verifier call.

The metric is verified draft rows per second (B*K per step); emitted tokens
per second is reported beside it. Inputs are synthetic and seeded (random
weights; no checkpoint or dataset) and larger than L2 per step. Timing: W
warm-up steps, then K steps bracketed by a barrier and device syncs, CUDA
events on the launching stream, max over ranks. One JSON line on rank 0.

--impl reference runs the float64 CPU oracle (the only other implementation
there is) on a bounded sample of the same workload on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from lossless_decoding_b200.inputs import (QWEN3_8B_HIDDEN, QWEN3_8B_PROJECTIONS,  # noqa: E402
                                           QWEN3_8B_VOCAB)

B64, K16, RANK, ALPHA = 64, 16, 128, 256.0
METRIC = "verified draft rows/s"
UNIT = "rows/s"


# B200 datasheet figures, reported beside the measured peaks so that every
# fraction can be read against either: HBM3e 8 TB/s, dense bf16 2.25 PFLOP/s.
DATASHEET = {"hbm": 8000.0, "bf16": 2250.0}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained"), "src": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "src": "fallback"}


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of those counters on the batched-decode workload; see the
# summaries in profiles/. A figure is reported only while the kernel source it was taken on
# is unchanged (first 16 hex digits of its sha256), else traffic is null.
MEASURED_TRAFFIC = {
    # dual_kernel: average of the step's four launches (63.6 + 3.2, 44.1 + 0.0,
    # 224.0 + 74.2, 130.1 + 0.1 MB read + written)
    ("batched_decode_b64_k16", "dual"): ("dualpath.cu", "33fb88aa9ae18da6", 134.84e6),
    # sample_drafts_kernel over the 64 x 16 q rows: 313.0 MB read + 3.6 MB written
    ("batched_decode_b64_k16", "draft"): ("draft_sample.cu", "9c3a8c794d39d5b7", 316.59e6),
    # stream 641.8 MB read + 3.4 MB written, draw 39.0 MB read, per verifier call
    ("batched_decode_b64_k16", "verify"): ("verify.cu", "85a3dfdf71983495", 684.24e6),
}


def measured_traffic(workload: str, kind: str):
    entry = MEASURED_TRAFFIC.get((workload, kind))
    if entry is None:
        return None
    import hashlib
    src, sha, nbytes = entry
    path = os.path.join(ROOT, "lossless_decoding_b200", "csrc", src)
    with open(path, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != sha:
            return None
    return nbytes


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's value (all ranks must call it, in the same
    order); the tensor lives on `device` (CUDA under NCCL, CPU under gloo)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_seeds(rank: int) -> tuple[int, int]:
    """(input seed, Philox key) of one replica. Replicas decode independent
    batches, so each draws its synthetic inputs and its acceptance / resampling
    uniforms from its own stream."""
    return 17 + rank, 1234 + rank


def whole_job_rate(rows_per_step: int, world: int, ms_step_max: float) -> float:
    """Rows per second over all ranks: each rank decodes rows_per_step rows per
    step, and the slowest rank's step time bounds the job."""
    return world * rows_per_step / (ms_step_max / 1e3)


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ---------------------------------------------------------------------------
# clocks sampled while the timed region runs
# ---------------------------------------------------------------------------


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML in a thread while
    the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, device: torch.device, period_s: float = 0.002):
        import threading
        self.period = period_s
        self.samples = []
        self.stop_evt = threading.Event()
        self.thread = None
        self.err = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report it instead of clocks
            self.nvml = None
            self.err = f"NVML unavailable: {e}"

    def _run(self):
        nv = self.nvml
        while not self.stop_evt.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                rs = get(self.h)
                self.samples.append((sm, rs))
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(self.period)

    def start(self):
        import threading
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no samples"]}
        self.stop_evt.set()
        self.thread.join(timeout=5)
        sm = [s for s, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items()
                          if r & bit})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm), "source": "NVML, polled during the timed region"}


# ---------------------------------------------------------------------------
# workloads on the device
# ---------------------------------------------------------------------------


def _dual_flops(M, d_in, d_out, r):
    return 2.0 * M * d_in * d_out + 2.0 * M * r * (d_in + d_out)


def layer_flops(M, layer):
    """Algorithmic FLOPs of one dual-path launch (all its projections)."""
    _, x, ds, *_ = layer
    return sum(_dual_flops(M, x.shape[1], d.W.shape[0], RANK) for d in ds)


# Projections that read the same activations run as one grouped launch.
PROJECTION_GROUPS = (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gate_up", ("gate", "up")),
                     ("down", ("down",)))


class BatchedDecode:
    """64 sequences x 16 drafts: 7 dual-path projections (4 launches) + verify."""

    name = "batched_decode_b64_k16"

    def __init__(self, dev, seed, philox_seed=1234):
        from lossless_decoding_b200 import api
        from lossless_decoding_b200.inputs import dualpath_inputs, verify_inputs
        self.philox_seed = philox_seed
        self.api = api
        self.B, self.K, self.V = B64, K16, QWEN3_8B_VOCAB
        self.M = self.B * self.K
        projs = {}
        for i, (name, d_in, d_out) in enumerate(QWEN3_8B_PROJECTIONS):
            projs[name] = dualpath_inputs(M=self.M, d_in=d_in, d_out=d_out, r=RANK, alpha=ALPHA,
                                          seed=seed * 100 + i, device=dev)
        # layers: one grouped launch each, (name, x, [inputs], [y_ar], [y_draft], workspace)
        self.layers = []
        for lname, members in PROJECTION_GROUPS:
            ds = [projs[m] for m in members]
            x = ds[0].x  # the members of a group read the same activations
            y_ars = [torch.empty((self.M, d.W.shape[0]), dtype=torch.bfloat16, device=dev)
                     for d in ds]
            y_drs = [torch.empty_like(y) for y in y_ars]
            need = sum(api.dualpath_workspace_bytes(self.M, d.x.shape[1], d.W.shape[0], RANK,
                                                    torch.bfloat16) for d in ds)
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
            self.layers.append((lname, x, ds, y_ars, y_drs, ws))
        self.v = verify_inputs(self.B, self.K, self.V, dtype="bf16", dist="normal", p_std=2.0,
                               sigma=1.0, seed=seed, device=dev)
        self.vws = torch.zeros(api.verify_workspace_bytes(self.B, self.K, self.V,
                                                          torch.bfloat16),
                               dtype=torch.uint8, device=dev)
        self.out = api.VerifyResult(
            torch.empty((self.B, self.K + 1), dtype=torch.int32, device=dev),
            torch.empty((self.B,), dtype=torch.int32, device=dev), None, None, None)
        self.gemm_flops = sum(layer_flops(self.M, layer) for layer in self.layers)
        self.verify_bytes = (self.B * (2 * self.K + 1) * self.V * 2 + self.B * self.K * 4
                             + self.B * (self.K + 2) * 4)
        self.launches_per_step = len(self.layers) + 3  # one dual-path launch each, verify: 3
        # bytes a step reads at least once (all distinct, so L2 cannot carry them)
        self.step_bytes = sum(x.numel() * 2 + sum(d.W.numel() * 2 + d.A.numel() * 2
                                                  + d.Bm.numel() * 2 for d in ds)
                              for _, x, ds, *_ in self.layers) + self.verify_bytes

    def step(self, seed_step, ev=None):
        api = self.api
        for i, (_, x, ds, y_ars, y_drs, ws) in enumerate(self.layers):
            if ev is not None:
                ev[0][i].record()
            api.dualpath_linear_grouped(x, [d.W for d in ds], [d.A for d in ds],
                                        [d.Bm for d in ds], [d.scale for d in ds],
                                        y_ars=y_ars, y_drafts=y_drs, workspace=ws)
            if ev is not None:
                ev[1][i].record()
        if ev is not None:
            ev[2].record()
        api.verify_block(self.v.p_logits, self.v.q_logits, self.v.draft_tokens,
                         seed=self.philox_seed,
                         step=seed_step, out=self.out, workspace=self.vws)
        if ev is not None:
            ev[3].record()

    def launch_flops(self, j):
        return layer_flops(self.M, self.layers[j])

    def extra_measurements(self, stream, reps=20):
        """Rows beyond the step: the on-device draft sampler over this
        workload's draft logits (B x K x V), timed alone with CUDA events on
        the launching stream (inputs larger than L2), against the HBM peak."""
        ids = torch.empty((self.B, self.K), dtype=torch.int32, device=self.out.out_tokens.device)
        for i in range(3):
            self.api.sample_drafts(self.v.q_logits, self.philox_seed, i, out=ids)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(reps):
            self.api.sample_drafts(self.v.q_logits, self.philox_seed, 100 + i, out=ids)
        b.record(stream)
        torch.cuda.synchronize()
        us = a.elapsed_time(b) * 1e3 / reps
        nbytes = self.v.q_logits.numel() * self.v.q_logits.element_size() + ids.numel() * 4
        gbs = nbytes / (us / 1e6) / 1e9
        peak = _peaks()["hbm"]
        # the verifier's calls back to back on the step's inputs: as in the
        # step, each call's stream launch sets up during the previous kernel
        # (the per-launch breakdown puts events between launches, which
        # serialises that set-up)
        for i in range(3):
            self.api.verify_block(self.v.p_logits, self.v.q_logits, self.v.draft_tokens,
                                  seed=self.philox_seed, step=i, out=self.out, workspace=self.vws)
        a.record(stream)
        for i in range(reps):
            self.api.verify_block(self.v.p_logits, self.v.q_logits, self.v.draft_tokens,
                                  seed=self.philox_seed, step=100 + i, out=self.out,
                                  workspace=self.vws)
        b.record(stream)
        torch.cuda.synchronize()
        us_v = a.elapsed_time(b) * 1e3 / reps
        gbs_v = self.verify_bytes / (us_v / 1e6) / 1e9
        return {"draft_sampler": {"kernel": "sample_drafts_kernel", "us": us, "achieved": gbs,
                                  "unit": "GB/s", "peak": peak, "frac": gbs / peak,
                                  "algorithmic_bytes": nbytes,
                                  "traffic": measured_traffic(self.name, "draft"),
                                  "rows": f"{self.B}x{self.K} rows of {self.V}"},
                "verifier_back_to_back": {"kernels": "verify_stream_kernel + verify_draw_kernel",
                                          "us": us_v, "achieved": gbs_v, "unit": "GB/s",
                                          "peak": peak, "frac": gbs_v / peak,
                                          "calls": reps, "algorithmic_bytes": self.verify_bytes}}

    def make_events(self):
        n = len(self.layers)
        mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        return ([mk() for _ in range(n)], [mk() for _ in range(n)], mk(), mk())

    def op_times(self, ev):
        gemm = sum(a.elapsed_time(b) for a, b in zip(ev[0], ev[1]))
        return gemm, ev[2].elapsed_time(ev[3])

    # host-resident inputs for the end-to-end measurement
    def host_inputs(self):
        pin = lambda t: t.cpu().pin_memory()  # noqa: E731
        xs = [pin(x) for _, x, *_ in self.layers]
        return xs, pin(self.v.p_logits), pin(self.v.q_logits), pin(self.v.draft_tokens)

    def e2e_step(self, host, step):
        xs, hp, hq, hx = host
        for (_, x, *_), hxv in zip(self.layers, xs):
            x.copy_(hxv, non_blocking=True)
        self.v.p_logits.copy_(hp, non_blocking=True)
        self.v.q_logits.copy_(hq, non_blocking=True)
        self.v.draft_tokens.copy_(hx, non_blocking=True)
        self.step(step)
        self.h_tok.copy_(self.out.out_tokens, non_blocking=True)
        self.h_len.copy_(self.out.accepted_len, non_blocking=True)

    def e2e_bytes(self, host):
        xs, hp, hq, hx = host
        h2d = sum(t.numel() * t.element_size() for t in xs) + sum(
            t.numel() * t.element_size() for t in (hp, hq, hx))
        d2h = self.out.out_tokens.numel() * 4 + self.out.accepted_len.numel() * 4
        self.h_tok = torch.empty_like(self.out.out_tokens, device="cpu").pin_memory()
        self.h_len = torch.empty_like(self.out.accepted_len, device="cpu").pin_memory()
        return h2d, d2h

    def emitted(self):
        return int((self.out.accepted_len.clamp(min=0) + 1).sum().item())

    def config(self):
        return {"workload": self.name, "B": self.B, "K": self.K, "V": self.V,
                "rows_M": self.M,
                "launches": [f"{n}:{x.shape[1]}->" + "+".join(str(d.W.shape[0]) for d in ds)
                             for n, x, ds, *_ in self.layers],
                "lora_rank": RANK, "lora_alpha": ALPHA, "logits": "bf16",
                "l2": f"inputs larger than L2: {self.step_bytes / 1e9:.2f} GB distinct per step",
                "global_batch": self.B, "parallelism": "replicas (one batch per GPU)"}


def tree_measure(api, stream, B, D, top_k, budget, V, reps=20, sets=4):
    """Time tree_draft (top-k + tree build) and tree_verify (node draws + walk)
    on the device: `sets` calls of each are captured in a CUDA graph (host
    overhead of the Python binding left out) and the graph is replayed `reps`
    times between CUDA events. The `sets` copies of the logits rotate so that
    the reads come from HBM (more than L2 in total)."""
    from lossless_decoding_b200.inputs import verify_inputs
    dev = torch.device("cuda", torch.cuda.current_device())
    N = api.tree_nodes(D, budget)
    qs = [verify_inputs(B, D, V, dtype="bf16", seed=50 + i, device=dev).q_logits
          for i in range(sets)]
    ps = [verify_inputs(B, N - 1, V, dtype="bf16", seed=60 + i, device=dev).p_logits
          for i in range(sets)]
    ws = torch.empty(api.tree_draft_workspace_bytes(B, D, V, top_k), dtype=torch.uint8,
                     device=dev)
    trees = [api.tree_draft(q, top_k, budget, workspace=ws) for q in qs]
    outs = [api.tree_verify(ps[i], trees[i], 1, 0) for i in range(sets)]
    torch.cuda.synchronize()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):  # warm-up on the capture's stream kind
        for i in range(sets):
            api.tree_draft(qs[i], top_k, budget, workspace=ws)
            api.tree_verify(ps[i], trees[i], 1, i, out=outs[i])
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    g_draft, g_verify = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_draft):
        for i in range(sets):
            api.tree_draft(qs[i], top_k, budget, workspace=ws)
    with torch.cuda.graph(g_verify):
        for i in range(sets):
            api.tree_verify(ps[i], trees[i], 1, i, out=outs[i])
    g_draft.replay()
    g_verify.replay()
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record(cur)
    for _ in range(reps):
        g_draft.replay()
    ev[1].record(cur)
    for _ in range(reps):
        g_verify.replay()
    ev[2].record(cur)
    torch.cuda.synchronize()
    us_d = ev[0].elapsed_time(ev[1]) * 1e3 / (reps * sets)
    us_v = ev[1].elapsed_time(ev[2]) * 1e3 / (reps * sets)
    rows = sum(int(t.n_nodes.sum()) for t in trees) / sets
    bytes_d = B * D * V * 2
    bytes_v = rows * V * 2
    peak = _peaks()["hbm"]
    del g_draft, g_verify
    return {"config": {"B": B, "D": D, "top_k": top_k, "budget": budget, "V": V,
                       "node_rows": N, "dtype": "bf16"},
            "timing": "CUDA graph of the calls, replayed between CUDA events",
            "draft_us": us_d, "draft_gbs": bytes_d / (us_d / 1e6) / 1e9,
            "verify_us": us_v, "verify_gbs": bytes_v / (us_v / 1e6) / 1e9,
            "verify_rows_in_use": rows, "peak_gbs": peak,
            "kernels": "tree_topk_part_kernel + tree_build_kernel (slab lists merged there); "
                       "sample_drafts_kernel (node rows) + tree_walk_kernel"}


class SingleSequence(BatchedDecode):
    """B = 1, K = 16: dual-path LM head over 17 rows, then verify its logits."""

    name = "qwen3_8b_b1"

    def __init__(self, dev, seed, philox_seed=1234):
        from lossless_decoding_b200 import api
        from lossless_decoding_b200.inputs import dualpath_inputs
        self.philox_seed = philox_seed
        self.api = api
        self.B, self.K, self.V = 1, K16, QWEN3_8B_VOCAB
        self.M = self.K + 1
        d = dualpath_inputs(M=self.M, d_in=QWEN3_8B_HIDDEN, d_out=self.V, r=RANK, alpha=ALPHA,
                            seed=seed, device=dev)
        y_ar = torch.empty((self.M, self.V), dtype=torch.bfloat16, device=dev)
        y_dr = torch.empty_like(y_ar)
        ws = torch.empty(api.dualpath_workspace_bytes(self.M, QWEN3_8B_HIDDEN, self.V, RANK,
                                                      torch.bfloat16), dtype=torch.uint8,
                         device=dev)
        self.layers = [("lm_head", d.x, [d], [y_ar], [y_dr], ws)]
        g = torch.Generator(device=dev).manual_seed(seed)
        self.drafts = torch.randint(0, self.V, (1, self.K), generator=g, device=dev,
                                    dtype=torch.int32)
        self.vws = torch.zeros(api.verify_workspace_bytes(1, self.K, self.V, torch.bfloat16),
                               dtype=torch.uint8, device=dev)
        self.out = api.VerifyResult(torch.empty((1, self.K + 1), dtype=torch.int32, device=dev),
                                    torch.empty((1,), dtype=torch.int32, device=dev), None, None,
                                    None)
        self.gemm_flops = _dual_flops(self.M, QWEN3_8B_HIDDEN, self.V, RANK)
        # 17 rows: HBM-bound on the weights; algorithmic bytes = W, A, Bm and x
        # read once, y_ar and y_draft written once
        self.gemm_bytes = ((d.W.numel() + d.A.numel() + d.Bm.numel() + d.x.numel()) * 2
                           + 2 * self.M * self.V * 2)
        self.verify_bytes = (2 * self.K + 1) * self.V * 2 + self.K * 4 + (self.K + 2) * 4
        self.launches_per_step = 4
        self.step_bytes = (d.x.numel() + d.W.numel() + d.A.numel() + d.Bm.numel()) * 2

    def step(self, seed_step, ev=None):
        api = self.api
        _, _, (d,), (y_ar,), (y_dr,), ws = self.layers[0]
        if ev is not None:
            ev[0][0].record()
        api.dualpath_linear(d.x, d.W, d.A, d.Bm, d.scale, y_ar=y_ar, y_draft=y_dr, workspace=ws)
        if ev is not None:
            ev[1][0].record()
            ev[2].record()
        p = y_ar.view(1, self.M, self.V)
        q = y_dr[: self.K].view(1, self.K, self.V)
        api.verify_block(p, q, self.drafts, seed=self.philox_seed, step=seed_step, out=self.out,
                         workspace=self.vws)
        if ev is not None:
            ev[3].record()

    def extra_measurements(self, stream, reps=20):
        """The LM head alone at exactly 16 rows (the K draft positions) and at
        the step's 17, timed over back-to-back calls (W, 1.24 GB, is larger
        than L2); and the tree sampler at this workload's batch: a block of 16
        (D = 15 positions after the AR-only first token), top-4 per position,
        the 16 best sequences kept (241 node rows)."""
        return {"lm_head_alone": self.lm_head_alone(stream, reps),
                "tree_sampler": tree_measure(self.api, stream, B=self.B, D=self.K - 1, top_k=4,
                                             budget=16, V=self.V, reps=reps)}

    def lm_head_alone(self, stream, reps):
        api = self.api
        _, _, (d,), (y_ar,), (y_dr,), ws = self.layers[0]
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        peak = _peaks()["hbm"]
        out = {}
        for rows in (16, self.M):
            x, ya, yd = d.x[:rows], y_ar[:rows], y_dr[:rows]
            need = api.dualpath_workspace_bytes(rows, QWEN3_8B_HIDDEN, self.V, RANK,
                                                torch.bfloat16)
            w = ws if ws.numel() >= need else torch.empty(need, dtype=torch.uint8,
                                                           device=ws.device)
            for _ in range(3):
                api.dualpath_linear(x, d.W, d.A, d.Bm, d.scale, y_ar=ya, y_draft=yd, workspace=w)
            a.record(stream)
            for _ in range(reps):
                api.dualpath_linear(x, d.W, d.A, d.Bm, d.scale, y_ar=ya, y_draft=yd, workspace=w)
            b.record(stream)
            torch.cuda.synchronize()
            us = a.elapsed_time(b) * 1e3 / reps
            nbytes = ((d.W.numel() + d.A.numel() + d.Bm.numel() + rows * QWEN3_8B_HIDDEN) * 2
                      + 2 * rows * self.V * 2)
            gbs = nbytes / (us / 1e6) / 1e9
            out[f"rows_{rows}"] = {"us": us, "achieved": gbs, "unit": "GB/s", "peak": peak,
                                   "frac": gbs / peak, "algorithmic_bytes": nbytes,
                                   "calls": reps}
        return out

    def host_inputs(self):
        _, x, *_ = self.layers[0]
        return [x.cpu().pin_memory()], self.drafts.cpu().pin_memory()

    def e2e_step(self, host, step):
        xs, hx = host
        self.layers[0][1].copy_(xs[0], non_blocking=True)
        self.drafts.copy_(hx, non_blocking=True)
        self.step(step)
        self.h_tok.copy_(self.out.out_tokens, non_blocking=True)
        self.h_len.copy_(self.out.accepted_len, non_blocking=True)

    def e2e_bytes(self, host):
        xs, hx = host
        h2d = xs[0].numel() * 2 + hx.numel() * 4
        self.h_tok = torch.empty_like(self.out.out_tokens, device="cpu").pin_memory()
        self.h_len = torch.empty_like(self.out.accepted_len, device="cpu").pin_memory()
        return h2d, (self.K + 2) * 4

    def config(self):
        c = super().config()
        c.update({"launches": [f"lm_head:{QWEN3_8B_HIDDEN}->{self.V}"], "rows_M": self.M,
                  "l2": "W of the LM head (1.24 GB) is larger than L2"})
        return c


class StackStep(BatchedDecode):
    """The whole Qwen3-8B-shaped draft-verify step at B = 64, K = 16.

    Rows: B x (K+1) = 1088 (each sequence's K drafted positions and its bonus
    row), sequence-major. Per layer (36, each with its own weights): the
    grouped q/k/v launch, o, the grouped gate/up launch and down, every
    projection with its rank-128 LoRA and the row gate closing the first row
    of each block (AR only). Stages are chained through the drafting pathway
    (o reads q's y_draft, down reads gate's, the next layer reads down's) as
    stand-ins for attention and the MLP nonlinearity, which are not on this
    path. Then the dual-path LM head 4096 -> 151936 (p = AR logits, q = draft
    logits) that also writes each row's softmax partials, the on-device draft
    sampler on q, and the verifier from those partials (it reads only the
    logits at the drafted ids and the rows of the final draw).
    """

    name = "qwen3_8b_stack_b64_k16"
    long_step = True  # ~20 ms of GEMMs per step: the sustained tensor peak applies
    verify_kernels = ("verify_decide_kernel + verify_draw_kernel (row statistics from the "
                      "LM head's epilogue; no streaming pass)")

    def __init__(self, dev, seed, philox_seed=1234):
        from lossless_decoding_b200 import api
        from lossless_decoding_b200.inputs import QWEN3_8B_LAYERS, dualpath_inputs
        self.philox_seed = philox_seed
        self.api = api
        self.B, self.K, self.V = B64, K16, QWEN3_8B_VOCAB
        self.M = self.B * (self.K + 1)
        M, H = self.M, QWEN3_8B_HIDDEN
        bf = torch.bfloat16
        self.x0 = (torch.randn(M, H, generator=torch.Generator(device=dev).manual_seed(seed),
                               device=dev)).to(bf)
        self.gate = torch.ones(M, dtype=torch.uint8, device=dev)
        self.gate.view(self.B, self.K + 1)[:, 0] = 0  # first position of each block: AR only
        shapes = {n: (i, o) for n, i, o in QWEN3_8B_PROJECTIONS}
        out = {n: (torch.empty(M, o, dtype=bf, device=dev), torch.empty(M, o, dtype=bf, device=dev))
               for n, (i, o) in shapes.items()}
        self.out = out
        self.layer_ws = []  # per layer: {projection: inputs}
        for layer in range(QWEN3_8B_LAYERS):
            ws = {}
            for j, (n, (i, o)) in enumerate(shapes.items()):
                # variance-preserving weights, so 36 chained stages keep
                # activations of unit scale; the adapter adds a small delta
                d = dualpath_inputs(M=1, d_in=i, d_out=o, r=RANK, alpha=ALPHA,
                                    w_std=i ** -0.5, b_std=0.004,
                                    seed=seed * 1000 + layer * 10 + j, device=dev)
                ws[n] = d
            self.layer_ws.append(ws)
        # logits of standard deviation about 2, as in the verifier's workload
        self.head = dualpath_inputs(M=1, d_in=H, d_out=self.V, r=RANK, alpha=ALPHA,
                                    w_std=2.0 * H ** -0.5, b_std=0.004,
                                    seed=seed * 1000 + 999, device=dev)
        self.p = torch.empty(M, self.V, dtype=bf, device=dev)
        self.q_all = torch.empty(M, self.V, dtype=bf, device=dev)
        # the LM head writes each row's softmax partials per 256-column tile;
        # the verifier merges those instead of streaming the logits again
        T = api.dualpath_stats_tiles(M, self.V)
        self.s_ar = torch.empty(M, T, 2, dtype=torch.float32, device=dev)
        self.s_dr = torch.empty(M, T, 2, dtype=torch.float32, device=dev)
        self.drafts = torch.empty(self.B, self.K, dtype=torch.int32, device=dev)
        need = max(api.dualpath_workspace_bytes(M, 12288, 12288, RANK, bf) * 3,
                   api.dualpath_workspace_bytes(M, H, self.V, RANK, bf))
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        self.vws = torch.zeros(api.verify_workspace_bytes(self.B, self.K, self.V, bf),
                               dtype=torch.uint8, device=dev)
        self.out_v = api.VerifyResult(
            torch.empty((self.B, self.K + 1), dtype=torch.int32, device=dev),
            torch.empty((self.B,), dtype=torch.int32, device=dev), None, None, None)
        # launches of one step: 4 per layer and the LM head (events bracket each)
        self.layers = []
        for _ in range(QWEN3_8B_LAYERS):
            self.layers += [("qkv", None), ("o", None), ("gate_up", None), ("down", None)]
        self.layers.append(("lm_head", None))
        lf = sum(_dual_flops(M, i, o, RANK) for _, i, o in QWEN3_8B_PROJECTIONS)
        self.gemm_flops = QWEN3_8B_LAYERS * lf + _dual_flops(M, H, self.V, RANK)
        # the verifier's algorithmic bytes with the LM head's statistics: the
        # partials of 2K+1 rows, the logits at the drafted ids, the p and q
        # rows of the final draw, drafts and outputs
        self.verify_bytes = (self.B * (2 * self.K + 1) * T * 8 + self.B * 2 * self.K * 2
                             + self.B * 2 * self.V * 2 + self.B * self.K * 4
                             + self.B * (self.K + 2) * 4)
        self.launches_per_step = len(self.layers) + 1 + 2  # + sampler, verifier: decide + draw
        self.step_bytes = 0

    def launch_flops(self, j):
        name = self.layers[j][0]
        if name == "lm_head":
            return _dual_flops(self.M, QWEN3_8B_HIDDEN, self.V, RANK)
        shapes = {n: (i, o) for n, i, o in QWEN3_8B_PROJECTIONS}
        members = dict(PROJECTION_GROUPS)[name]
        return sum(_dual_flops(self.M, *shapes[m], RANK) for m in members)

    def _dual(self, x, names, ws_layer):
        ds = [ws_layer[n] for n in names]
        self.api.dualpath_linear_grouped(x, [d.W for d in ds], [d.A for d in ds],
                                         [d.Bm for d in ds], [d.scale for d in ds],
                                         y_ars=[self.out[n][0] for n in names],
                                         y_drafts=[self.out[n][1] for n in names],
                                         workspace=self.ws, gate=self.gate)

    def step(self, seed_step, ev=None):
        api = self.api
        x = self.x0
        j = 0

        def mark(k):
            if ev is not None:
                ev[k][j].record()

        for ws_layer in self.layer_ws:
            for names, src in ((("q", "k", "v"), None), (("o",), "q"), (("gate", "up"), None),
                               (("down",), "gate")):
                inp = x if src is None else self.out[src][1]
                if names[0] == "gate":
                    inp = self.out["o"][1]
                mark(0)
                self._dual(inp, names, ws_layer)
                mark(1)
                j += 1
            x = self.out["down"][1]
        h = self.head
        mark(0)
        api.dualpath_linear_stats(x, h.W, h.A, h.Bm, h.scale, gate=self.gate, y_ar=self.p,
                                  y_draft=self.q_all, stats_ar=self.s_ar, stats_draft=self.s_dr,
                                  workspace=self.ws)
        mark(1)
        # the sampler reads the first K rows of each block of K + 1 in place
        api.sample_drafts(self.q_all.view(self.B, self.K + 1, self.V), self.philox_seed,
                          seed_step, out=self.drafts, num_drafts=self.K)
        if ev is not None:
            ev[2].record()
        api.verify_block_head(self.p, self.q_all, self.s_ar, self.s_dr, self.drafts,
                              seed=self.philox_seed, step=seed_step, out=self.out_v,
                              workspace=self.vws)
        if ev is not None:
            ev[3].record()

    def emitted(self):
        return int((self.out_v.accepted_len.clamp(min=0) + 1).sum().item())

    def extra_measurements(self, stream, reps=20):
        return {}

    def host_inputs(self):
        return [self.x0.cpu().pin_memory()], None

    def e2e_step(self, host, step):
        self.x0.copy_(host[0][0], non_blocking=True)
        self.step(step)
        self.h_tok.copy_(self.out_v.out_tokens, non_blocking=True)
        self.h_len.copy_(self.out_v.accepted_len, non_blocking=True)

    def e2e_bytes(self, host):
        h2d = host[0][0].numel() * host[0][0].element_size()
        d2h = self.out_v.out_tokens.numel() * 4 + self.out_v.accepted_len.numel() * 4
        self.h_tok = torch.empty_like(self.out_v.out_tokens, device="cpu").pin_memory()
        self.h_len = torch.empty_like(self.out_v.accepted_len, device="cpu").pin_memory()
        return h2d, d2h

    def config(self):
        from lossless_decoding_b200.inputs import QWEN3_8B_LAYERS
        return {"workload": self.name, "B": self.B, "K": self.K, "V": self.V,
                "rows_M": self.M, "layers": QWEN3_8B_LAYERS,
                "per_layer": "q+k+v, o, gate+up, down (grouped dual-path launches, row gate)",
                "then": ("dual-path LM head 4096->151936 writing row softmax partials, "
                         "draft sampler, verifier from those partials (no logit streaming)"),
                "lora_rank": RANK, "lora_alpha": ALPHA, "dtype": "bf16",
                "l2": "weights 13.9 GB per step, larger than L2",
                "global_batch": self.B, "parallelism": "replicas (one batch per GPU)"}


WORKLOADS = {c.name: c for c in (BatchedDecode, SingleSequence, StackStep)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


_SAMPLES = {}


def _oracle_inputs(workload: str, n_seq: int):
    """float64 inputs of a bounded sample (cached: generation is not timed)."""
    key = (workload, n_seq)
    if key in _SAMPLES:
        return _SAMPLES[key]
    from lossless_decoding_b200.inputs import dualpath_inputs, verify_inputs
    K, V = K16, QWEN3_8B_VOCAB
    if workload == "qwen3_8b_b1":
        projs, M = [("lm_head", QWEN3_8B_HIDDEN, V)], K + 1
    else:
        projs, M = list(QWEN3_8B_PROJECTIONS), n_seq * K
    dual = []
    for i, (_, d_in, d_out) in enumerate(projs):
        d = dualpath_inputs(M=M, d_in=d_in, d_out=d_out, r=RANK, alpha=ALPHA, seed=i)
        dual.append((d.x.double().numpy(), d.W.double().numpy(), d.A.double().numpy(),
                     d.Bm.double().numpy(), d.scale))
    v = verify_inputs(n_seq, K, V, dtype="bf16", seed=0)
    _SAMPLES[key] = (dual, v.p_logits.double().numpy(), v.q_logits.double().numpy(),
                     v.draft_tokens.numpy())
    return _SAMPLES[key]


def oracle_sample(workload: str, n_seq: int, step: int = 0):
    """Time the float64 oracle on n_seq sequences of the workload.

    The oracle's dual-path linear over the sample's rows of every projection,
    then its verifier over the sample's 2K+1 logit rows per sequence. Returns
    (seconds, verified rows).
    """
    import oracle
    dual, p, q, x = _oracle_inputs(workload, n_seq)
    t0 = time.perf_counter()
    for (xx, W, A, Bm, s) in dual:
        oracle.dualpath_linear(xx, W, A, Bm, s, round_t_to_bf16=True)
    oracle.verify_block(p, q, x, seed=1234, step=step)
    return time.perf_counter() - t0, n_seq * K16


def cpu_baseline(workload: str, min_seconds: float = 10.0, max_reps: int = 40):
    n_seq = 1 if workload == "qwen3_8b_b1" else 8
    secs = rows = reps = 0
    while reps < max_reps and (secs < min_seconds or reps == 0):
        s, r = oracle_sample(workload, n_seq, step=reps)
        secs, rows, reps = secs + s, rows + r, reps + 1
    return {"value": rows / secs, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": (f"{reps} x {n_seq} sequence(s), K={K16}: float64 oracle dual-path linear "
                       f"of every projection over the sample's rows, then the verifier over "
                       f"{n_seq}x{2 * K16 + 1} rows of {QWEN3_8B_VOCAB} logits; "
                       f"{secs:.1f} s of oracle time")}


def run_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    if args.workload == StackStep.name:
        print(json.dumps({"impl": "reference", "unavailable": "the float64 oracle of 36 layers "
                          "and the LM head does not fit a bounded host sample"}), flush=True)
        return 0
    if args.workload == SWEEP:
        print(json.dumps({"impl": "reference", "unavailable": "the sweep is a set of verifier "
                          "points, not one step a bounded oracle sample can stand for"}),
              flush=True)
        return 0
    n_seq = 1
    for i in range(args.warmup):
        oracle_sample(args.workload, n_seq, step=i)
    times = []
    rows = 0
    for i in range(args.steps):
        s, rows = oracle_sample(args.workload, n_seq, step=args.warmup + i)
        times.append(s)
    t = sum(times) / len(times)
    value = rows / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample_sequences": n_seq,
                       "note": "float64 CPU oracle on host cores, one bounded sample per step"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(),
                             "kind": "oracle",
                             "sample": f"{n_seq} sequence x K={K16} of {args.workload} per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the verifier sweep
# ---------------------------------------------------------------------------

SWEEP = "verifier_sweep"
SWEEP_B = (1, 8, 32, 64, 128, 256)
SWEEP_K = (4, 8, 16, 32)
SWEEP_DTYPES = ("bf16", "f32")
L2_BYTES = 126 * 2 ** 20


def sweep_points():
    pts = [(B, K, dt, 1.0) for dt in SWEEP_DTYPES for B in SWEEP_B for K in SWEEP_K]
    pts += [(B64, K16, "bf16", 0.25), (B64, K16, "bf16", 4.0)]
    return pts


def verify_algorithmic_bytes(B, K, V, esize):
    # every logit row once, the drafts, the outputs (tokens and lengths)
    return B * (2 * K + 1) * V * esize + B * K * 4 + B * (K + 2) * 4


def run_sweep(args):
    world, rank, local = _dist()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the kernels have no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from lossless_decoding_b200 import api
    from lossless_decoding_b200.inputs import verify_inputs
    peaks = _peaks()
    steps = max(3, min(args.steps, 10))
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(dev)
    clocks.start()
    points, tot_rows, tot_s = [], 0, 0.0
    for (B, K, dt, sigma) in sweep_points():
        V = QWEN3_8B_VOCAB
        v = verify_inputs(B, K, V, dtype=dt, dist="gumbel", sigma=sigma, seed=B * 100 + K,
                          device=dev)
        esize = v.p_logits.element_size()
        ws = torch.zeros(api.verify_workspace_bytes(B, K, V, v.p_logits.dtype),
                         dtype=torch.uint8, device=dev)
        out = api.VerifyResult(torch.empty((B, K + 1), dtype=torch.int32, device=dev),
                               torch.empty((B,), dtype=torch.int32, device=dev), None, None, None)
        nbytes = verify_algorithmic_bytes(B, K, V, esize)
        small = nbytes < 2 * L2_BYTES  # else the inputs alone exceed L2
        for i in range(args.warmup):
            api.verify_block(v.p_logits, v.q_logits, v.draft_tokens, seed=1234, step=i,
                             out=out, workspace=ws)
        ts = []
        for i in range(steps):
            if small:
                flush.fill_(i & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            api.verify_block(v.p_logits, v.q_logits, v.draft_tokens, seed=1234,
                             step=args.warmup + i, out=out, workspace=ws)
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1) / 1e3)
        t = statistics.median(ts)
        gbs = nbytes / t / 1e9
        acc = float(out.accepted_len.clamp(min=0).float().mean().item())
        points.append({"B": B, "K": K, "dtype": dt, "sigma": sigma, "us": t * 1e6,
                       "GBps": gbs, "frac": gbs / peaks["hbm"], "rows_per_s": B * K / t,
                       "mean_accepted": acc, "logit_bytes": B * (2 * K + 1) * V * esize,
                       "l2_flushed": small})
        tot_rows += B * K
        tot_s += t
        del v, ws, out
        torch.cuda.empty_cache()
    clk = clocks.stop()
    if rank == 0:
        big = [p for p in points if p["logit_bytes"] >= 4 * L2_BYTES]
        line = {
            "metric": METRIC, "value": tot_rows / tot_s, "unit": UNIT, "n_gpus": 1,
            "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / len(points),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16+f32", "data": "synthetic (seeded Gumbel logits, top-20 boosted)",
            "config": {"workload": SWEEP, "V": QWEN3_8B_VOCAB, "points": len(points),
                       "l2": "flushed before each timed call where a point's bytes are "
                             "below 2x L2; larger points exceed L2 by themselves",
                       "value": "all points' rows / the sum of their median call times"},
            "roofline": {"kernel": "verify_stream_kernel + verify_draw_kernel", "bound": "hbm",
                         "peak": peaks["hbm"], "unit": "GB/s",
                         "frac_min_large": min(p["frac"] for p in big) if big else None,
                         "frac_median_large": (statistics.median(p["frac"] for p in big)
                                               if big else None),
                         "large": "points with at least 4x L2 of logits",
                         "peak_kind": f"HBM copy, {peaks['src']}"},
            "sweep": points, "clocks": clk, "gpu_launches": 2 * len(points) * steps,
        }
        print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------


def run_ours(args):
    world, rank, local = _dist()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the kernels have no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    from lossless_decoding_b200 import api

    input_seed, philox_seed = replica_seeds(rank)
    wl = WORKLOADS[args.workload](dev, seed=input_seed, philox_seed=philox_seed)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    def rank_max(x: float) -> float:
        return max_over_ranks(x, world, dev)

    for i in range(args.warmup):
        wl.step(i)
    api.device_fault_flags(clear=True)
    barrier()

    # ---- timed region: K steps back to back (kernels may overlap their
    # set-up with the previous kernel's tail, so no events between them) ----
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev)
    clocks.start()
    barrier()
    t0.record(stream)
    for i in range(args.steps):
        wl.step(args.warmup + i)
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    ms_step = rank_max(ms_total / args.steps)
    emitted = wl.emitted()

    # ---- per-launch breakdown: the same steps with CUDA events around every
    # launch on the launching stream (for the roofline of each kernel) ----
    n_bd = max(1, min(args.steps, 20))
    events = [wl.make_events() for _ in range(n_bd)]
    barrier()
    for i in range(n_bd):
        wl.step(args.warmup + args.steps + i, events[i])
    barrier()
    gemm_ms = [wl.op_times(e)[0] for e in events]
    ver_ms = [wl.op_times(e)[1] for e in events]
    faults = api.device_fault_flags(clear=True)
    extra = wl.extra_measurements(stream) if hasattr(wl, "extra_measurements") else {}

    rows_per_step = wl.B * wl.K
    value = whole_job_rate(rows_per_step, world, ms_step)
    peaks = _peaks()
    gemm_avg = sum(gemm_ms) / len(gemm_ms)
    ver_avg = sum(ver_ms) / len(ver_ms)
    gemm_tflops = wl.gemm_flops / (gemm_avg / 1e3) / 1e12
    per_launch = {}  # by launch name (summed over a step's launches of that name)
    for j, layer in enumerate(wl.layers):
        us = 1e3 * sum(e[0][j].elapsed_time(e[1][j]) for e in events) / len(events)
        acc = per_launch.setdefault(layer[0], [0.0, 0.0])
        acc[0] += us
        acc[1] += wl.launch_flops(j)
    per_proj = {n: {"us": round(us, 2), "tflops": round(fl / (us / 1e6) / 1e12, 1)}
                for n, (us, fl) in per_launch.items()}
    ver_gbs = wl.verify_bytes / (ver_avg / 1e3) / 1e9
    dominant_gemm = gemm_avg >= ver_avg
    gemm_kernel = "dual_kernel (T tiles, x W^T and T Bm^T, one persistent launch)"
    gemm_bytes = getattr(wl, "gemm_bytes", None)
    if gemm_bytes is None:  # tensor-core bound: FLOPs against the dense bf16 peak
        # a step of many milliseconds of back-to-back GEMMs runs under the power
        # cap: its peak is the sustained one; a short step takes the burst peak
        sustained = getattr(wl, "long_step", False) and peaks.get("bf16_sustained")
        peak_tf = peaks["bf16_sustained"] if sustained else peaks["bf16"]
        kind = "sustained (seconds-long loop under the power cap)" if sustained else "burst"
        roof_gemm = {"kernel": gemm_kernel, "bound": "tensor", "achieved": gemm_tflops,
                     "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": gemm_tflops / peak_tf,
                     "frac_burst": gemm_tflops / peaks["bf16"],
                     "frac_datasheet": gemm_tflops / DATASHEET["bf16"],
                     "traffic": measured_traffic(args.workload, "dual"),
                     "peak_kind": f"bf16 dense {kind}, {peaks['src']}; datasheet 2250 TFLOP/s",
                     "algorithmic_per_launch": wl.gemm_flops / len(wl.layers),
                     "ms_per_step": gemm_avg}
    else:  # few rows: the stream of W bounds it, bytes against the HBM peak
        gemm_gbs = gemm_bytes / (gemm_avg / 1e3) / 1e9
        roof_gemm = {"kernel": gemm_kernel, "bound": "hbm", "achieved": gemm_gbs,
                     "peak": peaks["hbm"], "unit": "GB/s", "frac": gemm_gbs / peaks["hbm"],
                     "frac_datasheet": gemm_gbs / DATASHEET["hbm"],
                     "traffic": measured_traffic(args.workload, "dual"),
                     "peak_kind": f"HBM copy, {peaks['src']}; datasheet 8000 GB/s",
                     "algorithmic_per_launch": gemm_bytes / len(wl.layers),
                     "tflops": gemm_tflops, "ms_per_step": gemm_avg}
    roof_ver = {"kernel": getattr(wl, "verify_kernels",
                                  "verify_stream_kernel + verify_draw_kernel"),
                "bound": "hbm", "achieved": ver_gbs,
                "peak": peaks["hbm"], "unit": "GB/s", "frac": ver_gbs / peaks["hbm"],
                "frac_datasheet": ver_gbs / DATASHEET["hbm"],
                "traffic": measured_traffic(args.workload, "verify"),
                "peak_kind": f"HBM copy, {peaks['src']}; datasheet 8000 GB/s",
                "algorithmic_per_launch": wl.verify_bytes, "ms_per_step": ver_avg}

    # ---- end to end: host buffers, copies inside the timed region ----
    host = wl.host_inputs()
    h2d, d2h = wl.e2e_bytes(host)
    e_steps = max(2, min(args.steps, 10))
    for i in range(2):
        wl.e2e_step(host, i)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e_steps):
        wl.e2e_step(host, 100 + i)
    e1.record(stream)
    barrier()
    e2e_ms = rank_max(e0.elapsed_time(e1) / e_steps)
    e2e_value = whole_job_rate(rows_per_step, world, e2e_ms)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded random weights, activations, logits)",
            "config": wl.config(),
            "emitted_tokens_per_s": world * emitted / (ms_step / 1e3),
            "gemm_tflops": gemm_tflops, "verify_gbs": ver_gbs, "gemm_per_launch": per_proj,
            "roofline": roof_gemm if dominant_gemm else roof_ver,
            "roofline_verify" if dominant_gemm else "roofline_gemm":
                roof_ver if dominant_gemm else roof_gemm,
            "gpu_launches": wl.launches_per_step * args.steps,
            "clocks": clk,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "device_fault_flags": faults,
            **extra,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = (cpu_baseline(args.workload)
                                    if args.workload != StackStep.name else
                                    {"value": None, "reason": "the float64 oracle of 36 layers and "
                                     "the LM head does not fit a bounded host sample"})
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + [SWEEP],
                    default="batched_decode_b64_k16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == SWEEP:
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
