"""Grouped dual-path launches (several projections of one x) on a B200.

A grouped launch must give every projection exactly what a separate
uno_dualpath_linear call gives (same tiles, same arithmetic: bit for bit; the
shapes here are small enough that no launch splits its last round along K)
and both must match the float64 oracle within the dual-path criterion
(tests/parity.py). Covers the swapped (M <= 256) and the CTA-pair (M > 256)
layouts, bf16 and f32, ragged output widths and projections without y_ar.
"""

import numpy as np
import pytest
import torch

import oracle
from lossless_decoding_b200.inputs import dualpath_inputs
from tests.parity import assert_dualpath_close, widen

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_decoding_b200 import api as A
    return A


def _projections(M, d_in, d_outs, r, dtype, seed):
    """One x, and per projection its own W, A, Bm (seeded generators)."""
    ds = [dualpath_inputs(M=M, d_in=d_in, d_out=o, r=r, alpha=2.0 * r, dtype=dtype,
                          seed=seed + 7 * g, device=DEV) for g, o in enumerate(d_outs)]
    x = ds[0].x
    return x, ds


CASES = [
    (520, 256, (512, 128, 136), 64, "bf16"),   # pair layout, ragged widths, 3 projections
    (1024, 512, (1024, 256, 256), 128, "bf16"),  # q/k/v proportions
    (300, 128, (256, 264), 32, "bf16"),         # gate/up-like pair, ragged M
    (17, 512, (384, 128, 64), 128, "bf16"),     # swapped layout (bonus-row decode)
    (200, 256, (128, 200, 72, 64), 16, "bf16"),  # four projections, swapped
    (520, 260, (300, 100), 36, "f32"),          # TF32 pair layout
    (40, 300, (100, 36, 8), 20, "f32"),         # TF32 swapped
]


@pytest.mark.parametrize("M,d_in,d_outs,r,dtype", CASES)
def test_grouped_equals_separate_calls_bit_for_bit(api, M, d_in, d_outs, r, dtype):
    x, ds = _projections(M, d_in, d_outs, r, dtype, seed=M + d_in)
    y_ars, y_drs = api.dualpath_linear_grouped(x, [d.W for d in ds], [d.A for d in ds],
                                               [d.Bm for d in ds], [d.scale for d in ds])
    torch.cuda.synchronize()
    for g, d in enumerate(ds):
        ya, yd = api.dualpath_linear(x, d.W, d.A, d.Bm, d.scale)
        torch.cuda.synchronize()
        assert torch.equal(y_ars[g], ya), f"projection {g}: y_ar differs from a separate call"
        assert torch.equal(y_drs[g], yd), f"projection {g}: y_draft differs from a separate call"


@pytest.mark.parametrize("M,d_in,d_outs,r,dtype", [CASES[0], CASES[3], CASES[5]])
def test_grouped_parity_with_oracle(api, M, d_in, d_outs, r, dtype):
    x, ds = _projections(M, d_in, d_outs, r, dtype, seed=3 * M + d_in)
    y_ars, y_drs = api.dualpath_linear_grouped(x, [d.W for d in ds], [d.A for d in ds],
                                               [d.Bm for d in ds], [d.scale for d in ds])
    torch.cuda.synchronize()
    for g, d in enumerate(ds):
        ref_ar, ref_dr, _ = oracle.dualpath_linear(
            widen(x), widen(d.W), widen(d.A), widen(d.Bm), d.scale,
            round_t_to_bf16=(x.dtype == torch.bfloat16))
        assert_dualpath_close(y_ars[g], ref_ar)
        assert_dualpath_close(y_drs[g], ref_dr)


def test_grouped_without_adapter_and_partial_outputs(api):
    x, ds = _projections(520, 256, (512, 136, 128), 64, "bf16", seed=11)
    Ws, As, Bms, sc = [d.W for d in ds], [d.A for d in ds], [d.Bm for d in ds], [d.scale for d in ds]
    y_ars, y_drs = api.dualpath_linear_grouped(x, Ws, As, Bms, sc, want_draft=False)
    torch.cuda.synchronize()
    assert all(y is None for y in y_drs)
    for g, d in enumerate(ds):
        ya, _ = api.dualpath_linear(x, d.W, d.A, d.Bm, d.scale, want_draft=False)
        torch.cuda.synchronize()
        assert torch.equal(y_ars[g], ya)
    # y_ar skipped for one projection only (a NULL y_ar for that projection)
    y_ars, y_drs = api.dualpath_linear_grouped(x, Ws, As, Bms, sc, want_ar=[True, False, True])
    torch.cuda.synchronize()
    assert y_ars[1] is None
    for g, d in enumerate(ds):
        ya, yd = api.dualpath_linear(x, d.W, d.A, d.Bm, d.scale)
        torch.cuda.synchronize()
        assert torch.equal(y_drs[g], yd)
        if y_ars[g] is not None:
            assert torch.equal(y_ars[g], ya)


def _sampled_rows(M, seed, n=64, tail=16):
    rows = np.random.default_rng(seed).choice(M - tail, size=n, replace=False)
    return np.sort(np.concatenate([rows, np.arange(M - tail, M)]))


# The grouped launches the benchmark times, at their full sizes: batched decode
# (64 x 16 = 1024 rows, q/k/v and gate/up of a Qwen3-8B-shaped layer, rank 128,
# alpha 256) and the whole-stack step (64 x 17 = 1088 rows, every launch with
# the row gate closing the first position of each block of 17, weights of
# standard deviation d_in^-1/2 and Bm of 0.004).
FULL_SIZE = [
    ("qkv_1024", 1024, 4096, (4096, 1024, 1024), False),
    ("gate_up_1024", 1024, 4096, (12288, 12288), False),
    ("qkv_1088_gated", 1088, 4096, (4096, 1024, 1024), True),
    ("o_1088_gated", 1088, 4096, (4096,), True),
    ("gate_up_1088_gated", 1088, 4096, (12288, 12288), True),
    ("down_1088_gated", 1088, 12288, (4096,), True),
]


@pytest.mark.parametrize("name,M,d_in,d_outs,gated", FULL_SIZE, ids=[c[0] for c in FULL_SIZE])
def test_benchmarked_grouped_launches_sampled_rows(api, name, M, d_in, d_outs, gated):
    kw = dict(w_std=d_in ** -0.5, b_std=0.004) if gated else {}
    ds = [dualpath_inputs(M=M, d_in=d_in, d_out=o, r=128, alpha=256.0, seed=M + 11 * g + d_in,
                          device=DEV, **kw) for g, o in enumerate(d_outs)]
    x = ds[0].x
    gate = None
    g_np = None
    if gated:
        g_np = np.ones(M, dtype=np.uint8)
        g_np[::17] = 0
        gate = torch.from_numpy(g_np).to(DEV)
    y_ars, y_drs = api.dualpath_linear_grouped(x, [d.W for d in ds], [d.A for d in ds],
                                               [d.Bm for d in ds], [d.scale for d in ds],
                                               gate=gate)
    torch.cuda.synchronize()
    rows = _sampled_rows(M, seed=M + d_in)
    ri = torch.from_numpy(rows).to(DEV)
    for g, d in enumerate(ds):
        ref_ar, ref_dr, _ = oracle.dualpath_linear(
            widen(x[ri]), widen(d.W), widen(d.A), widen(d.Bm), d.scale, round_t_to_bf16=True,
            gate=None if g_np is None else g_np[rows])
        assert_dualpath_close(y_ars[g][ri], ref_ar)
        assert_dualpath_close(y_drs[g][ri], ref_dr)
        if gated:
            closed = torch.from_numpy(g_np == 0).to(DEV)
            assert torch.equal(y_drs[g][closed], y_ars[g][closed])
    assert api.device_fault_flags() == 0
    del ds, y_ars, y_drs
    torch.cuda.empty_cache()
