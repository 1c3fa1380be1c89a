"""Parity of the CUDA block verifier with the float64 oracle (needs a B200).

Inputs come from lossless_decoding_b200.inputs (seeded); the oracle gets the
same bytes widened exactly to float64 and the same (seed, step). Token ids
and accepted lengths must match bit for bit outside near-tie bands; the
counts of excluded near-ties are reported (tests/parity.py).
"""

import numpy as np
import pytest
import torch
from scipy import stats

import oracle
from lossless_decoding_b200.inputs import verify_inputs
from tests.parity import VerifyReport, compare_verify, report, widen

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_decoding_b200 import api as A
    return A


def _run(api, v, seed, step, probs=True, lse=True):
    res = api.verify_block(v.p_logits.to(DEV), v.q_logits.to(DEV), v.draft_tokens.to(DEV),
                           seed=seed, step=step, want_probs=probs, want_lse=lse)
    torch.cuda.synchronize()
    return res


def _oracle(v, seed, step):
    return oracle.verify_block(widen(v.p_logits), widen(v.q_logits), v.draft_tokens.numpy(),
                               seed=seed, step=step)


@pytest.mark.parametrize("B,K,V,dtype,dist,sigma", [
    (1, 8, 4096, "f32", "normal", 0.5),        # tiny configuration
    (3, 1, 1, "bf16", "normal", 1.0),          # V = 1
    (4, 3, 7, "f32", "normal", 1.0),           # V below one vector
    (5, 4, 9, "bf16", "normal", 2.0),          # ragged head / tail
    (2, 16, 4097, "bf16", "normal", 1.0),      # odd V: rows not 16-byte aligned
    (7, 5, 4097, "f32", "gumbel", 1.0),
    (3, 32, 20000, "bf16", "gumbel", 4.0),     # K = 32, low acceptance
    (16, 16, 32000, "bf16", "gumbel", 0.25),   # high acceptance, many bonus draws
    (64, 4, 1000, "f32", "normal", 0.5),
])
def test_parity_small(api, B, K, V, dtype, dist, sigma):
    for seed, step in ((0, 0), (123, 7)):
        v = verify_inputs(B, K, V, dtype=dtype, dist=dist, sigma=sigma, seed=seed + B + K)
        rep = compare_verify(_run(api, v, seed, step), _oracle(v, seed, step))
        assert rep.compared + rep.accept_ties + rep.draw_ties == B
    assert api.device_fault_flags() == 0


def test_workspace_is_reusable_and_calls_are_independent(api):
    v = verify_inputs(8, 6, 3001, dtype="bf16", seed=5)
    # start from garbage: the kernels must not depend on the workspace contents
    ws = torch.full((api.verify_workspace_bytes(8, 6, 3001, torch.bfloat16),), 0xA5,
                    dtype=torch.uint8, device=DEV)
    outs = []
    for step in range(4):
        res = api.verify_block(v.p_logits.to(DEV), v.q_logits.to(DEV), v.draft_tokens.to(DEV),
                               seed=9, step=step, workspace=ws, want_probs=True)
        torch.cuda.synchronize()
        compare_verify(res, _oracle(v, 9, step))
        outs.append(res.out_tokens.cpu())
    again = api.verify_block(v.p_logits.to(DEV), v.q_logits.to(DEV), v.draft_tokens.to(DEV),
                             seed=9, step=0, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(again.out_tokens.cpu(), outs[0])


def test_outputs_stay_in_bounds(api):
    B, K, V = 5, 7, 999
    v = verify_inputs(B, K, V, dtype="f32", seed=2)
    canary = -77
    big_out = torch.full((B * (K + 1) + 64,), canary, dtype=torch.int32, device=DEV)
    big_len = torch.full((B + 64,), canary, dtype=torch.int32, device=DEV)
    big_p = torch.full((B * K + 64,), 1e30, dtype=torch.float32, device=DEV)
    big_q = torch.full((B * K + 64,), 1e30, dtype=torch.float32, device=DEV)
    big_l = torch.full((B * (2 * K + 1) + 64,), 1e30, dtype=torch.float32, device=DEV)
    out = api.VerifyResult(big_out[: B * (K + 1)].view(B, K + 1), big_len[:B],
                           big_p[: B * K].view(B, K), big_q[: B * K].view(B, K),
                           big_l[: B * (2 * K + 1)].view(B, 2 * K + 1))
    api.verify_block(v.p_logits.to(DEV), v.q_logits.to(DEV), v.draft_tokens.to(DEV), 1, 1, out=out)
    torch.cuda.synchronize()
    assert torch.all(big_out[B * (K + 1):] == canary)
    assert torch.all(big_len[B:] == canary)
    assert torch.all(big_p[B * K:] == 1e30) and torch.all(big_q[B * K:] == 1e30)
    assert torch.all(big_l[B * (2 * K + 1):] == 1e30)
    compare_verify(out, _oracle(v, 1, 1))


def test_special_cases(api):
    B, K, V = 32, 4, 300
    g = torch.Generator().manual_seed(0)
    p = torch.randn(B, K + 1, V, generator=g) * 2
    # identical draft -> everything accepted, bonus from p_K
    x = torch.randint(0, V, (B, K), generator=g, dtype=torch.int32)
    res = api.verify_block(p.to(DEV), p[:, :K].contiguous().to(DEV), x.to(DEV), 3, 0)
    torch.cuda.synchronize()
    assert torch.all(res.accepted_len.cpu() == K)
    ref = oracle.verify_block(p.double().numpy(), p[:, :K].double().numpy(), x.numpy(), 3, 0)
    assert np.array_equal(res.out_tokens.cpu().numpy(), ref["out_tokens"])
    # masked vocabulary: -inf logits never emitted
    pm = p.clone()
    pm[:, :, : V // 2] = float("-inf")
    q = torch.randn(B, K, V, generator=g)
    xq = torch.randint(0, V, (B, K), generator=g, dtype=torch.int32)
    res = api.verify_block(pm.to(DEV), q.to(DEV), xq.to(DEV), 4, 0)
    torch.cuda.synchronize()
    out = res.out_tokens.cpu()
    n = res.accepted_len.cpu()
    for b in range(B):
        assert out[b, n[b]] >= V // 2
    compare_verify(res, oracle.verify_block(pm.double().numpy(), q.double().numpy(), xq.numpy(),
                                            4, 0), check_probs=False)
    # invalid draft ids flag their sequence only
    xb = x.clone()
    xb[3, 1] = V
    xb[7, 0] = -5
    res = api.verify_block(p.to(DEV), q.to(DEV), xb.to(DEV), 5, 0)
    torch.cuda.synchronize()
    n = res.accepted_len.cpu()
    assert n[3] == -1 and n[7] == -1 and torch.all(res.out_tokens.cpu()[[3, 7]] == -1)
    compare_verify(res, oracle.verify_block(p.double().numpy(), q.double().numpy(), xb.numpy(),
                                            5, 0), check_probs=False)


def test_chisquare_on_device(api):
    V, K, B = 8, 3, 1 << 20
    rng = np.random.default_rng(42)
    # float32-representable logits, so the oracle and the device see the same values
    p = rng.normal(0, 1.2, size=(K + 1, V)).astype(np.float32).astype(np.float64)
    q = (p[:K] + rng.normal(0, 1.0, size=(K, V))).astype(np.float32).astype(np.float64)
    Qp = np.exp(q - q.max(1, keepdims=True))
    Qp /= Qp.sum(1, keepdims=True)
    x = np.stack([rng.choice(V, size=B, p=Qp[i]) for i in range(K)], axis=1).astype(np.int32)
    pt = torch.tensor(p, dtype=torch.float32).expand(B, K + 1, V).contiguous()
    qt = torch.tensor(q, dtype=torch.float32).expand(B, K, V).contiguous()
    res = api.verify_block(pt.to(DEV), qt.to(DEV), torch.from_numpy(x).to(DEV), 77, 0)
    torch.cuda.synchronize()
    out = res.out_tokens.cpu().numpy()
    n = res.accepted_len.cpu().numpy()
    P = np.exp(p - p.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    assert stats.chisquare(np.bincount(out[:, 0], minlength=V), P[0] * B).pvalue > 1e-3
    for j in range(K + 1):
        sel = out[n >= j, j]
        assert stats.chisquare(np.bincount(sel, minlength=V), P[j] * sel.size).pvalue > 1e-3
    # and bit-exact against the oracle on a slice (same counters: rows 0..2^16-1)
    s = 1 << 16
    ref = oracle.verify_block(np.broadcast_to(p, (s, K + 1, V)), np.broadcast_to(q, (s, K, V)),
                              x[:s], 77, 0)
    sub = api.VerifyResult(res.out_tokens[:s], res.accepted_len[:s], None, None, None)
    rep = compare_verify(sub, ref, check_probs=False)
    assert rep.compared > 0.99 * s


def _sampled_full_size(api, B, K, V, dtype, dist, sigma, n_check, seed, step):
    """Full-size call; the oracle checks a seeded sample of sequences."""
    v = verify_inputs(B, K, V, dtype=dtype, dist=dist, sigma=sigma, seed=seed, device=DEV)
    res = api.verify_block(v.p_logits, v.q_logits, v.draft_tokens, seed, step, want_probs=True,
                           want_lse=True)
    torch.cuda.synchronize()
    idx = np.sort(np.random.default_rng(seed).choice(B, size=min(n_check, B), replace=False))
    u_acc, u_smp = oracle.uniforms_for_block(B, K, seed, step)
    totals = np.zeros(5, dtype=np.int64)
    for c0 in range(0, idx.size, 16):  # bounded host memory for the float64 oracle
        sel = idx[c0:c0 + 16]
        it = torch.from_numpy(sel).to(DEV)
        ref = oracle.verify_block_u(widen(v.p_logits[it]), widen(v.q_logits[it]),
                                    v.draft_tokens[it].cpu().numpy(), u_acc[sel], u_smp[sel])
        sub = api.VerifyResult(res.out_tokens[it], res.accepted_len[it], res.p_at_draft[it],
                               res.q_at_draft[it], res.row_lse[it])
        r = compare_verify(sub, ref)
        totals += np.array([r.rows, r.compared, r.accept_ties, r.draw_ties, r.invalid])
    rep = VerifyReport(*[int(t) for t in totals])
    # properties that hold for every sequence
    n = res.accepted_len.cpu()
    assert torch.all((n >= 0) & (n <= K))
    out = res.out_tokens.cpu()
    assert torch.all(out[torch.arange(B), n] >= 0)
    return rep


def _floor(n: int) -> int:
    """Sequences that must be compared token for token out of n checked. The
    draw band of tests/parity.py leaves about 5% of full-vocabulary draws as
    near ties: 90% for samples of 32 and more; a few sequences fewer for the
    small samples of single sweep points (their sum is held to 90% by
    test_parity_verifier_sweep_compares_ninety_percent)."""
    return int(np.ceil(0.9 * n)) if n >= 32 else n - max(1, n // 4)


@pytest.mark.parametrize("B,K,dtype,dist,sigma,n_check", [
    (1, 16, "bf16", "normal", 1.0, 1),       # Qwen3-8B single sequence
    (64, 16, "bf16", "normal", 1.0, 64),     # batched decode B=64, K=16 (full oracle)
    (256, 32, "f32", "gumbel", 4.0, 32),     # largest sweep point (10 GB of logits)
    (128, 8, "bf16", "gumbel", 0.25, 32),
])
def test_parity_full_vocabulary(api, B, K, dtype, dist, sigma, n_check):
    rep = _sampled_full_size(api, B, K, 151936, dtype, dist, sigma, n_check, seed=B + K, step=3)
    n = min(n_check, B)
    report(f"full vocabulary B={B} K={K} {dtype} {dist} sigma={sigma}", rep)
    assert rep.compared + rep.accept_ties + rep.draw_ties == n
    assert rep.compared >= _floor(n), f"only {rep.compared} of {n} sequences compared"
    assert api.device_fault_flags() == 0
    torch.cuda.empty_cache()


def _sweep_cases():
    """Every (B, K) of the verifier sweep (B in {1..256}, K in {4..32}), V = 151936,
    Gumbel-like logits with a boosted top-20; dtype and the draft noise sigma
    cycle so that each value of each meets several B and K."""
    cases = []
    sigmas = (0.25, 1.0, 4.0)
    for i, B in enumerate((1, 8, 32, 64, 128, 256)):
        for j, K in enumerate((4, 8, 16, 32)):
            dtype = "bf16" if (i + j) % 2 == 0 else "f32"
            cases.append((B, K, dtype, sigmas[(i + 2 * j) % 3]))
    return cases


@pytest.mark.parametrize("B,K,dtype,sigma", _sweep_cases())
def test_parity_verifier_sweep(api, B, K, dtype, sigma):
    n = min(B, 16)
    rep = _sampled_full_size(api, B, K, 151936, dtype, "gumbel", sigma, n, seed=7 * B + K,
                             step=B + K)
    report(f"sweep B={B} K={K} {dtype} sigma={sigma}", rep)
    assert rep.compared + rep.accept_ties + rep.draw_ties == n
    assert rep.compared >= _floor(n), f"only {rep.compared} of {n} sequences compared"
    assert api.device_fault_flags() == 0
    torch.cuda.empty_cache()


def test_parity_verifier_sweep_compares_ninety_percent():
    """Over every point of the verifier sweep run in this session, at least 90%
    of the checked sequences are compared token for token (the rest are near
    ties of the derived band)."""
    from tests.parity import REPORTS
    sweep = [r for name, r in REPORTS if name.startswith("sweep ")]
    if len(sweep) < len(_sweep_cases()):
        pytest.skip("the sweep did not run in full in this session")
    rows = sum(r.rows for r in sweep)
    compared = sum(r.compared for r in sweep)
    assert compared >= 0.9 * rows, f"{compared} of {rows} sweep sequences compared"
