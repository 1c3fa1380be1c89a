"""Pins of the oracle's dual-pathway linear and of its bfloat16 helpers.

The dual-pathway linear follows "Unlocking Lossless Speedups in LLMs via
Discrete Diffusion" (picx.dev summary, Methodology / Architecture; paperglide
reader, The Uno Framework): the frozen AR weight W is shared, drafting adds a
rank-r LoRA adapter scaled by alpha/r, verification uses W alone. The pins:
a hand-worked example (tests/golden/dualpath_hand.json), brute-force loops in
plain Python, and invariants (zero adapter, zero scale, zero-padded rank,
the parameter count the pages print).
"""

import json
import os

import numpy as np
import pytest

from oracle import bf16_bits_to_f64, dualpath_linear, round_to_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_hand_example():
    with open(os.path.join(GOLDEN, "dualpath_hand.json")) as f:
        g = json.load(f)
    y_ar, y_dr, T = dualpath_linear(g["x"], g["W"], g["A"], g["Bm"], g["scale"],
                                    round_t_to_bf16=False)
    assert y_ar.tolist() == g["y_ar"]
    assert T.tolist() == g["T"]
    assert y_dr.tolist() == g["y_draft"]
    # Every value there is a small integer, so bf16 rounding of T changes nothing.
    _, y_dr2, _ = dualpath_linear(g["x"], g["W"], g["A"], g["Bm"], g["scale"],
                                  round_t_to_bf16=True)
    assert y_dr2.tolist() == g["y_draft"]


def _loops(x, W, A, Bm, s):
    M, d_in = len(x), len(x[0])
    d_out, r = len(W), len(A)
    y_ar = [[sum(x[m][k] * W[o][k] for k in range(d_in)) for o in range(d_out)]
            for m in range(M)]
    T = [[s * sum(x[m][k] * A[j][k] for k in range(d_in)) for j in range(r)] for m in range(M)]
    y_dr = [[y_ar[m][o] + sum(T[m][j] * Bm[o][j] for j in range(r)) for o in range(d_out)]
            for m in range(M)]
    return np.array(y_ar), np.array(y_dr), np.array(T)


@pytest.mark.parametrize("M,d_in,d_out,r", [(1, 1, 1, 1), (3, 5, 4, 2), (4, 7, 9, 3)])
def test_bruteforce_loops(M, d_in, d_out, r):
    rng = np.random.default_rng(M * 100 + d_in)
    x, W = rng.normal(size=(M, d_in)), rng.normal(size=(d_out, d_in))
    A, Bm = rng.normal(size=(r, d_in)), rng.normal(size=(d_out, r))
    s = 1.75
    ref = _loops(x.tolist(), W.tolist(), A.tolist(), Bm.tolist(), s)
    got = dualpath_linear(x, W, A, Bm, s, round_t_to_bf16=False)
    for a, b in zip(got, ref):
        assert np.allclose(a, b, rtol=1e-13, atol=1e-13)


def test_zero_adapter_and_zero_scale_leave_the_ar_path():
    rng = np.random.default_rng(0)
    x, W = rng.normal(size=(6, 16)), rng.normal(size=(8, 16))
    A, Bm = rng.normal(size=(4, 16)), rng.normal(size=(8, 4))
    y_ar, y_dr, _ = dualpath_linear(x, W, A, np.zeros_like(Bm), 2.0, True)
    assert np.array_equal(y_ar, y_dr)
    y_ar, y_dr, _ = dualpath_linear(x, W, A, Bm, 0.0, True)
    assert np.array_equal(y_ar, y_dr)


def test_zero_padded_rank_changes_nothing():
    rng = np.random.default_rng(1)
    x, W = rng.normal(size=(5, 12)), rng.normal(size=(7, 12))
    A, Bm = rng.normal(size=(3, 12)), rng.normal(size=(7, 3))
    A8 = np.concatenate([A, np.zeros((5, 12))])
    B8 = np.concatenate([Bm, np.zeros((7, 5))], axis=1)
    a = dualpath_linear(x, W, A, Bm, 3.0, True)
    b = dualpath_linear(x, W, A8, B8, 3.0, True)
    assert np.array_equal(a[0], b[0]) and np.allclose(a[1], b[1], rtol=1e-14, atol=1e-14)


def test_rounded_adapter_input_is_bf16_and_close():
    rng = np.random.default_rng(2)
    x, W = rng.normal(size=(9, 32)), rng.normal(size=(5, 32))
    A, Bm = rng.normal(size=(16, 32)), rng.normal(size=(5, 16))
    _, _, T = dualpath_linear(x, W, A, Bm, 2.0, round_t_to_bf16=True)
    _, _, Te = dualpath_linear(x, W, A, Bm, 2.0, round_t_to_bf16=False)
    assert np.array_equal(round_to_bf16(T), T)
    assert np.all(np.abs(T - Te) <= 2.0**-8 * np.abs(Te) * (1 + 1e-12))


def test_lora_parameter_count_matches_the_pages():
    # The pages give 0.35B extra parameters for rank-128 adapters on every
    # projection of the 8B model (picx.dev summary, Main Results; Table 2
    # context). Qwen3-8B shapes: 36 layers of q,o 4096->4096; k,v 4096->1024;
    # gate,up 4096->12288; down 12288->4096. A LoRA adapter of rank r on a
    # d_in->d_out projection holds r*(d_in + d_out) parameters.
    from lossless_decoding_b200.inputs import QWEN3_8B_LAYERS, QWEN3_8B_PROJECTIONS
    r = 128
    per_layer = sum(r * (di + do) for _, di, do in QWEN3_8B_PROJECTIONS)
    total = per_layer * QWEN3_8B_LAYERS
    assert abs(total / 1e9 - 0.35) < 0.005


def test_bf16_golden_values():
    with open(os.path.join(GOLDEN, "bf16_values.json")) as f:
        g = json.load(f)
    for x, want in g["round"]:
        assert round_to_bf16(np.array([x]))[0] == want, x
    for bits, want in g["bits"]:
        assert bf16_bits_to_f64(np.array([bits], dtype=np.uint16))[0] == want, bits


def test_bf16_rounding_is_nearest():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 100, size=20000)
    r = round_to_bf16(x)
    # Representable: exactly 8 significant bits.
    f, _ = np.frexp(r)
    assert np.all(np.ldexp(f, 8) == np.rint(np.ldexp(f, 8)))
    # Nearest: error at most half a spacing (spacing = 2^(e-8) for |x| in [2^(e-1), 2^e)).
    _, e = np.frexp(x)
    assert np.all(np.abs(r - x) <= np.ldexp(0.5, e - 8))


def test_gate_rows_are_ar_only_and_open_rows_unchanged():
    """Gated LoRA (reader page, "The Psi-Speculative Sampler"): a closed row's
    draft output is its AR output exactly; an open row is the ungated result."""
    rng = np.random.default_rng(5)
    M, d_in, d_out, r = 7, 24, 16, 8
    x = rng.standard_normal((M, d_in))
    W = rng.standard_normal((d_out, d_in)) * 0.1
    A = rng.standard_normal((r, d_in)) * 0.1
    Bm = rng.standard_normal((d_out, r)) * 0.1
    gate = np.array([0, 1, 1, 0, 1, 0, 1], dtype=np.uint8)
    y_ar, y_dr, T = dualpath_linear(x, W, A, Bm, 2.0, False, gate=gate)
    y_ar0, y_dr0, T0 = dualpath_linear(x, W, A, Bm, 2.0, False)
    assert np.array_equal(y_ar, y_ar0)
    for m in range(M):
        if gate[m]:
            assert np.array_equal(y_dr[m], y_dr0[m]) and np.array_equal(T[m], T0[m])
        else:
            assert np.array_equal(y_dr[m], y_ar[m]) and not np.any(T[m])
    # brute force for one open row, written out as loops
    m = 2
    for j in range(d_out):
        want = sum(x[m, k] * W[j, k] for k in range(d_in))
        want += sum(2.0 * sum(x[m, k] * A[i, k] for k in range(d_in)) * Bm[j, i]
                    for i in range(r))
        assert abs(y_dr[m, j] - want) < 1e-12
    # all-open gate is the ungated call; all-closed makes the adapter vanish
    assert np.array_equal(dualpath_linear(x, W, A, Bm, 2.0, False, gate=np.ones(M))[1], y_dr0)
    assert np.array_equal(dualpath_linear(x, W, A, Bm, 2.0, False, gate=np.zeros(M))[1], y_ar0)
