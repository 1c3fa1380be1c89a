"""Grouped dual-path launches (several projections of one x) on a B200.

A grouped launch must give every projection exactly what a separate
uno_dualpath_linear call gives (same tiles, same arithmetic: bit for bit; the
shapes here are small enough that no launch splits its last round along K)
and both must match the float64 oracle within the dual-path criterion
(tests/parity.py). Covers the swapped (M <= 256) and the CTA-pair (M > 256)
layouts, bf16 and f32, ragged output widths and projections without y_ar.
"""

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
