"""Comparison rules between the CUDA path and the float64 oracle.

Token ids and accepted lengths must match exactly, except where the oracle's
decision lies within a near-tie band (the device cannot decide it the same way
for certain):
  * an accept test with |u - p/q| < 1e-5 (the stated criterion); the row is
    not compared from that position on;
  * a verifier draw whose threshold u' * total lies within
    TAU_DRAW * (total + q_res) of a CDF boundary of the oracle, q_res the q
    mass on the residual's support (0 for a draw from p);
  * a draft draw whose threshold u * total lies within
    TAU_DRAFT * sqrt(sum of squared weights) of a CDF boundary of the oracle.
Probabilities must match within 1e-5 absolute.

The verifier's draw band follows from its arithmetic. A token weight is
2^(x log2 e - L) on the SFU (relative error at most 1.46e-7, measured over
every float in [-0.5, 1] against float64) with the argument from three
float32 FMA roundings (each at most 2^-24 of |argument|); a 16-byte vector's
weights are summed as a float32 tree (three roundings), longer sums in
float64; the row normalisers come from the streaming pass's float32 sums.
Per-token errors e_i move the comparison of the running sum C_v with
u' C_total by (1 - u') sum_{i<=v} e_i - u' sum_{i>v} e_i, a common factor
on all weights cancels, and the normalisers' ratio enters through the q
mass of the residual's support, q_res. Replaying these roundings in float32
over rows shaped like the test workloads (151936 tokens, Gaussian and
boosted-Gumbel logits, 128 draws, the SFU error injected at its measured
maximum and each normaliser perturbed by 1e-7), the comparison moved by at
most 1.1e-7 (total + q_res); the band is three times that:
TAU_DRAW * (total + q_res).

The draft sampler's band follows from its arithmetic (pass 1: per-lane sums
of 2^(x log2 e - m) with m the lane's running maximum, one FMA and the SFU
per logit, float32 pair trees and accumulation, each lane's sum rescaled to
the warp's maximum and added in float64; pass 2: chunk sums rescaled to the
row's maximum in float64; pass 3: the chosen chunk's weights by the SFU,
summed in float64). The per-token relative errors (the SFU's, the argument's
and the float32 sums' roundings) are uncorrelated across tokens, so their
weighted sum, which is what moves a comparison, grows like the row's spread
sqrt(sum_i w_i^2), not like its total: replayed in float32 over rows of 151936
tokens (Gaussian and boosted-Gumbel logits of spread 0.25 to 4, float32 and
bfloat16, the SFU's error injected at its maximum), the comparison moved by
at most 2.68e-7 of the spread on every workload, while relative to the total
the moves ranged from 4e-9 (diffuse rows) to 2.0e-7 (concentrated ones). The
band is three times that, rounded up: TAU_DRAFT * sqrt(sum_i w_i^2).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

ACCEPT_TIE = 1e-5
TAU_DRAW = 3e-7
TAU_DRAFT = 8.1e-7  # draft sampler, times the row's spread: see the module docstring
PROB_ATOL = 1e-5


def widen(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16/f32 tensor (CPU)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


@dataclass
class VerifyReport:
    rows: int
    compared: int
    accept_ties: int
    draw_ties: int
    invalid: int


def compare_verify(gpu, ref, check_probs: bool = True) -> VerifyReport:
    """Assert the CUDA verifier agrees with the oracle; return tie counts."""
    n_g = gpu.accepted_len.cpu().numpy()
    out_g = gpu.out_tokens.cpu().numpy()
    n_o = ref["accepted_len"]
    out_o = ref["out_tokens"]
    B, K1 = out_o.shape
    K = K1 - 1
    ratio, u = ref["ratio"], ref["u_acc"]
    acc_ties = draw_ties = compared = invalid = 0
    for b in range(B):
        if n_o[b] < 0:
            invalid += 1
            assert n_g[b] == -1 and np.all(out_g[b] == -1), f"row {b}: invalid drafts not flagged"
            continue
        last = min(n_o[b], K - 1)
        tie = np.abs(u[b, : last + 1] - ratio[b, : last + 1]) < ACCEPT_TIE
        if tie.any():
            acc_ties += 1
            first = int(np.argmax(tie))
            # decisions before the tie must still agree
            assert n_g[b] >= first, f"row {b}: rejected at {n_g[b]} before tie at {first}"
            assert np.array_equal(out_g[b, :first], out_o[b, :first])
            continue
        assert n_g[b] == n_o[b], f"row {b}: accepted {n_g[b]} vs oracle {n_o[b]}"
        n = n_o[b]
        assert np.array_equal(out_g[b, :n], out_o[b, :n])
        assert np.all(out_g[b, n + 1:] == -1)
        t, lo, hi, tot = ref["cdf_t"][b], ref["cdf_prev"][b], ref["cdf_at"][b], ref["cdf_total"][b]
        tau = TAU_DRAW * (tot + ref["cdf_qres"][b])
        if min(t - lo, hi - t) < tau:
            draw_ties += 1
            continue
        assert out_g[b, n] == out_o[b, n], f"row {b}: token {out_g[b, n]} vs oracle {out_o[b, n]}"
        compared += 1
    if check_probs and gpu.p_at_draft is not None:
        valid = n_o >= 0
        for name in ("p_at_draft", "q_at_draft"):
            g = getattr(gpu, name).cpu().numpy()[valid]
            err = np.abs(g - ref[name][valid]).max() if valid.any() else 0.0
            assert err < PROB_ATOL, f"{name} max abs error {err}"
    if gpu.row_lse is not None:
        g = gpu.row_lse.cpu().numpy()
        err = np.abs(g - ref["row_lse"]).max()
        # lse = log Z: an absolute error of e in lse is a relative error e in Z.
        assert err < 2e-5 * max(1.0, np.abs(ref["row_lse"]).max()), f"row_lse error {err}"
    rep = VerifyReport(B, compared, acc_ties, draw_ties, invalid)
    return rep


# Comparison counts of the tests of a session, printed at its end (conftest).
REPORTS: list = []


def report(name: str, rep: VerifyReport) -> VerifyReport:
    """Record a test's comparison counts for the session summary."""
    REPORTS.append((name, rep))
    return rep


def rel_err_normwise(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def assert_dualpath_close(got: torch.Tensor, ref: np.ndarray, tol: float = 2e-2):
    """Normwise max relative error (the stated criterion) plus an elementwise
    bound |y - ref| <= tol*|ref| + tol*rms(ref)."""
    g = widen(got)
    assert g.shape == ref.shape
    assert np.all(np.isfinite(g))
    e = rel_err_normwise(g, ref)
    assert e < tol, f"normwise relative error {e}"
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    bad = np.abs(g - ref) > tol * np.abs(ref) + tol * rms
    assert not bad.any(), f"{int(bad.sum())} elements outside the elementwise bound"
    return e


def compare_drafts(got: np.ndarray, ids: np.ndarray, det: dict) -> tuple[int, int]:
    """Drafted ids of the CUDA sampler against the oracle: equal except draws
    whose threshold lies within TAU_DRAFT * spread of a CDF boundary (spread =
    sqrt of the row's sum of squared weights). Returns (compared, ties)."""
    got = np.asarray(got)
    assert got.shape == ids.shape
    t, lo, hi, tot = det["threshold"], det["c_prev"], det["c_at"], det["total"]
    tie = np.minimum(t - lo, hi - t) < TAU_DRAFT * det["spread"]
    tie &= ids >= 0
    bad = (got != ids) & ~tie
    assert not bad.any(), f"{int(bad.sum())} drafted ids differ, first at {np.argwhere(bad)[0]}"
    return int((~tie).sum()), int(tie.sum())
