"""Parity of the LM head with row statistics and of the verifier that uses
them (the LM head fused with the verifier's softmax statistics), on a B200.

* ``dualpath_linear_stats`` writes exactly the outputs of the gated dual-path
  call (bit for bit), and its per-tile partials reproduce each row's
  logsumexp of the stored logits (float64 oracle softmax) within 2e-5, and
  each tile's maximum exactly (times log2 e, in float32);
* ``verify_block_head`` on the LM head's outputs agrees with the float64
  oracle verifier run on p = y_ar rows and q = the first K y_draft rows of
  each block, with the same near-tie accounting as the plain verifier;
  row_lse, p(x_i) and q(x_i) within the plain verifier's tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_decoding_b200.inputs import dualpath_inputs
from tests.parity import VerifyReport, compare_verify, report, widen

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LOG2E = 1.4426950408889634


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_decoding_b200 import api as A
    return A


def _head(M, d_in, d_out, r, dtype, seed, w_std=0.05):
    d = dualpath_inputs(M=M, d_in=d_in, d_out=d_out, r=r, alpha=2.0 * r, dtype=dtype,
                        w_std=w_std, seed=seed, device=DEV)
    return d


def _lse_from_stats(st):
    """Row logsumexp (natural log) from [rows, T, 2] partials, in float64."""
    m = st[..., 0].astype(np.float64)
    z = st[..., 1].astype(np.float64)
    top = m.max(axis=1, keepdims=True)
    tot = (z * np.exp2(m - top)).sum(axis=1)
    return (top[:, 0] + np.log2(tot)) * np.log(2.0)


@pytest.mark.parametrize("M,d_in,d_out,dtype", [
    (300, 256, 1000, "bf16"),      # ragged rows and a ragged last column tile
    (520, 512, 3000, "f32"),       # the TF32 path
    (1088, 1024, 20000, "bf16"),   # 64 blocks of 17 rows
])
def test_stats_match_outputs(api, M, d_in, d_out, dtype):
    d = _head(M, d_in, d_out, 64, dtype, seed=M + d_out)
    gate = torch.ones(M, dtype=torch.uint8, device=DEV)
    gate[::17] = 0
    y_ar, y_dr, s_ar, s_dr = api.dualpath_linear_stats(d.x, d.W, d.A, d.Bm, d.scale, gate=gate)
    ref_ar, ref_dr = api.dualpath_linear(d.x, d.W, d.A, d.Bm, d.scale, gate=gate)
    torch.cuda.synchronize()
    assert torch.equal(y_ar, ref_ar) and torch.equal(y_dr, ref_dr)
    T = api.dualpath_stats_tiles(M, d_out)
    assert T == (d_out + 255) // 256 and tuple(s_ar.shape) == (M, T, 2)
    for y, st in ((y_ar, s_ar), (y_dr, s_dr)):
        yw = widen(y)
        stn = st.cpu().numpy()
        _, lse = oracle.softmax_rows(yw)
        got = _lse_from_stats(stn)
        assert np.abs(got - lse).max() < 2e-5 * max(1.0, np.abs(lse).max())
        # each tile's reference is its largest stored value times log2 e
        pad = T * 256 - d_out
        tiles = np.pad(yw, ((0, 0), (0, pad)), constant_values=-np.inf).reshape(M, T, 256)
        want_m = (tiles.max(axis=2) * LOG2E).astype(np.float32)
        assert np.allclose(stn[..., 0], want_m, rtol=1e-6, atol=0)


@pytest.mark.parametrize("M,d_in,d_out,dtype", [
    (17, 256, 1000, "bf16"),       # one block of 17 rows: BN = 32, ragged column tile
    (200, 512, 3000, "f32"),       # BN = 256, the TF32 path
    (68, 1024, 151936, "bf16"),    # four blocks over the full vocabulary: every CTA busy
])
def test_swapped_stats_match_outputs(api, M, d_in, d_out, dtype):
    """Small batches (swapped operands): one partial per CTA, merged over the
    CTA's column tiles; slots of CTAs the launch did not start are empty."""
    d = _head(M, d_in, d_out, 64, dtype, seed=M + d_out)
    gate = torch.ones(M, dtype=torch.uint8, device=DEV)
    gate[::17] = 0
    y_ar, y_dr, s_ar, s_dr = api.dualpath_linear_stats(d.x, d.W, d.A, d.Bm, d.scale, gate=gate)
    ref_ar, ref_dr = api.dualpath_linear(d.x, d.W, d.A, d.Bm, d.scale, gate=gate)
    torch.cuda.synchronize()
    assert torch.equal(y_ar, ref_ar) and torch.equal(y_dr, ref_dr)
    T = api.dualpath_stats_tiles(M, d_out)
    assert T == 148 and tuple(s_ar.shape) == (M, T, 2)
    for y, st in ((y_ar, s_ar), (y_dr, s_dr)):
        yw = widen(y)
        stn = st.cpu().numpy()
        _, lse = oracle.softmax_rows(yw)
        got = _lse_from_stats(stn)
        assert np.abs(got - lse).max() < 2e-5 * max(1.0, np.abs(lse).max())
        # every reference is the largest stored value of some of the row's
        # columns (times log2 e); together they reach the row's maximum
        m = stn[..., 0]
        z = stn[..., 1]
        empty = m == -np.inf
        assert np.all(z[empty] == 0) and np.all(z[~empty] >= 1 - 1e-6)
        want_top = (yw.max(axis=1) * LOG2E).astype(np.float32)
        assert np.allclose(m.max(axis=1), want_top, rtol=1e-6, atol=0)
    assert api.device_fault_flags() == 0


def _check_head_verify(api, B, K, V, d_in, dtype, seed, step, n_check=None, sigma_w=0.05):
    M = B * (K + 1)
    d = _head(M, d_in, V, 64, dtype, seed=seed, w_std=sigma_w)
    gate = torch.ones(M, dtype=torch.uint8, device=DEV)
    gate.view(B, K + 1)[:, 0] = 0  # the first position of each block: AR weights only
    y_ar, y_dr, s_ar, s_dr = api.dualpath_linear_stats(d.x, d.W, d.A, d.Bm, d.scale, gate=gate)
    q = y_dr.view(B, K + 1, V)[:, :K].contiguous()
    drafts = api.sample_drafts(q, seed, step)
    res = api.verify_block_head(y_ar, y_dr, s_ar, s_dr, drafts, seed, step, want_probs=True,
                                want_lse=True)
    torch.cuda.synchronize()
    idx = np.arange(B) if n_check is None else \
        np.sort(np.random.default_rng(seed).choice(B, size=n_check, replace=False))
    u_acc, u_smp = oracle.uniforms_for_block(B, K, seed, step)
    totals = np.zeros(5, dtype=np.int64)
    for c0 in range(0, idx.size, 16):
        sel = idx[c0:c0 + 16]
        it = torch.from_numpy(sel).to(DEV)
        p = widen(y_ar.view(B, K + 1, V)[it])
        qq = widen(q[it])
        ref = oracle.verify_block_u(p, qq, drafts[it].cpu().numpy(), u_acc[sel], u_smp[sel])
        sub = api.VerifyResult(res.out_tokens[it], res.accepted_len[it], res.p_at_draft[it],
                               res.q_at_draft[it], res.row_lse[it])
        r = compare_verify(sub, ref)
        totals += np.array([r.rows, r.compared, r.accept_ties, r.draw_ties, r.invalid])
    rep = VerifyReport(*[int(t) for t in totals])
    assert rep.compared + rep.accept_ties + rep.draw_ties == idx.size
    n = res.accepted_len.cpu()
    assert torch.all((n >= 0) & (n <= K))
    # the plain verifier on the same logits decides the same (up to near ties)
    plain = api.verify_block(y_ar.view(B, K + 1, V), q, drafts, seed, step)
    torch.cuda.synchronize()
    same = (plain.accepted_len == res.accepted_len).float().mean().item()
    assert same > 0.95
    return rep


@pytest.mark.parametrize("B,K,V,d_in,dtype", [
    (32, 8, 3000, 256, "bf16"),
    (20, 15, 5000, 512, "f32"),     # the TF32 path, V not a multiple of 256
    (12, 8, 5000, 256, "f32"),      # 108 rows, swapped, TF32
])
def test_verify_head_parity(api, B, K, V, d_in, dtype):
    for seed, step in ((5, 0), (41, 9)):
        rep = _check_head_verify(api, B, K, V, d_in, dtype, seed, step)
        report(f"LM head B={B} K={K} V={V} {dtype} seed={seed}", rep)
        assert rep.compared >= int(np.ceil(0.9 * B)) - 1


def test_verify_head_single_sequence(api):
    """One sequence (17 rows, swapped operands) over eight steps: at least
    seven of the eight blocks compared token for token."""
    tot = np.zeros(5, dtype=np.int64)
    for step in range(8):
        r = _check_head_verify(api, 1, 16, 20000, 512, "bf16", seed=11, step=step)
        tot += np.array([r.rows, r.compared, r.accept_ties, r.draw_ties, r.invalid])
    rep = VerifyReport(*[int(t) for t in tot])
    report("LM head B=1 K=16 V=20000 bf16, 8 steps", rep)
    assert rep.compared >= 7


def test_verify_head_qwen3_lm_head(api):
    """The LM head of the batched step: 64 blocks of 17 rows, 4096 -> 151936,
    bf16; the oracle checks 32 sequences, and at least 90% of them (less one)
    must be compared token for token outside the derived near-tie band."""
    rep = _check_head_verify(api, 64, 16, 151936, 4096, "bf16", seed=7, step=3, n_check=32,
                             sigma_w=0.03)
    report("LM head B=64 K=16 V=151936 bf16", rep)
    assert rep.compared >= 28, f"only {rep.compared} of 32 sequences compared"
    assert api.device_fault_flags() == 0
