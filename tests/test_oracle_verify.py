"""Pins of the oracle's block verifier (linear Psi-Spec sampler).

The pages ("Unlocking Lossless Speedups in LLMs via Discrete Diffusion",
paperglide reader, The Psi-Speculative Sampler and Sampler Extensions; picx.dev
summary, Methodology / Psi-Speculative Sampler) claim the sampler preserves
the AR distribution exactly. These tests pin the oracle to that claim and to
closed forms, never to itself:

* brute force: every draft tuple of a tiny vocabulary, every outcome, with
  the accept and sampling uniforms integrated EXACTLY over their 2^24-point
  grid (binary search on the oracle's own monotone decisions), checking
  P(reach j, prefix, out_j = v) = P(reach j, prefix) * p_j(v), and the two
  routes min(p, q) (accepted draft) and max(0, p - q) (residual);
* a chi-square test on 10^6 Philox-driven draws;
* the mean accepted length sum_j prod_{i<j} (1 - TV_i) (the blockwise TV
  quantity of the training objective, whose complement is the per-position
  acceptance probability);
* hand-worked K=1, V=2 cases (tests/golden/verify_k1_v2.json) and special
  cases with known outcomes.
"""

import itertools
import json
import os

import numpy as np
import pytest
from scipy import special, stats

import oracle.uno_oracle as oracle_mod
from oracle import softmax_rows, uniforms_for_block, verify_block

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
G = 1 << 24  # size of the uniform grid


def _lib_softmax(logits):
    return special.softmax(np.asarray(logits, dtype=np.float64), axis=-1)


# --------------------------------------------------------------------------
# exact integration over the 24-bit uniform grid
# --------------------------------------------------------------------------


def _grid_search(pred, batch):
    """Per row, the smallest g in [0, G] with pred(g) False (pred monotone:
    True below a threshold, False from it on); G if pred is always True."""
    lo = np.zeros(batch, dtype=np.int64)
    hi = np.full(batch, G, dtype=np.int64)
    while np.any(lo < hi):
        mid = (lo + hi) // 2
        t = pred(np.minimum(mid, G - 1))
        active = lo < hi
        lo = np.where(active & t, mid + 1, lo)
        hi = np.where(active & ~t, mid, hi)
    return lo


def _exact_outcomes(p_logits, q_logits):
    """Outcome probabilities of the oracle over all draft tuples.

    Returns a list of (emitted tuple, route, probability), where probability
    includes the draft weight prod_i q_i(x_i) and the exact grid measure of
    the uniforms that produce this outcome.
    """
    K1, V = p_logits.shape
    K = K1 - 1
    tuples = np.array(list(itertools.product(range(V), repeat=K)), dtype=np.int64)
    T = tuples.shape[0]
    P = _lib_softmax(p_logits)
    Q = _lib_softmax(q_logits)
    pb = np.broadcast_to(p_logits, (T, K1, V)).copy()
    qb = np.broadcast_to(q_logits, (T, K, V)).copy()

    # c[t, i]: grid points of u_i accepted at position i for tuple t.
    c = np.zeros((T, K), dtype=np.int64)
    for i in range(K):
        def pred(g, i=i):
            ua = np.zeros((T, K))
            ua[:, i] = g * 2.0**-24
            res = oracle_mod.verify_block_u(pb, qb, tuples, ua, np.zeros((T, K1)))
            return res["accepted_len"] > i
        c[:, i] = _grid_search(pred, T)

    # wres[t, j, v]: grid points of u'_j giving token v when position j is
    # the first rejection (only meaningful where rejection is possible).
    wres = np.zeros((T, K1, V), dtype=np.int64)
    can_reject = np.zeros((T, K), dtype=bool)
    for j in range(K1):
        # bound[t, v] = #{g : y(g) < v}; widths are differences.
        TT = T * (V + 1)
        tt = np.repeat(np.arange(T), V + 1)
        vv = np.tile(np.arange(V + 1), T)
        ua = np.zeros((TT, K))
        if j < K:
            ua[:, j] = 1.0 - 2.0**-24  # reject at j when q_j(x_j) > p_j(x_j)
        probe = oracle_mod.verify_block_u(pb[tt], qb[tt], tuples[tt], ua, np.zeros((TT, K1)))
        ok = probe["accepted_len"] == j

        def pred(g, j=j):
            us = np.zeros((TT, K1))
            us[:, j] = g * 2.0**-24
            res = oracle_mod.verify_block_u(pb[tt], qb[tt], tuples[tt], ua, us)
            return res["out_tokens"][:, j] < vv

        bound = _grid_search(pred, TT).reshape(T, V + 1)
        bound[:, V] = G
        wres[:, j, :] = np.diff(bound, axis=1)
        if j < K:
            can_reject[:, j] = ok.reshape(T, V + 1)[:, 0]

    qw = np.prod(Q[np.arange(K)[None, :], tuples], axis=1)  # draft weight
    outcomes = []
    for t in range(T):
        x = tuples[t]
        reach = qw[t]
        for n in range(K1):
            if n < K:
                p_rej = (G - c[t, n]) / G
                if p_rej > 0:
                    assert can_reject[t, n]
                    for y in range(V):
                        if wres[t, n, y]:
                            outcomes.append((tuple(x[:n]) + (y,), "residual",
                                             reach * p_rej * wres[t, n, y] / G))
                reach *= c[t, n] / G
            else:
                for y in range(V):
                    if wres[t, K, y]:
                        outcomes.append((tuple(x) + (y,), "bonus", reach * wres[t, K, y] / G))
    return outcomes, P, Q


def _check_lossless(p_logits, q_logits):
    K1, V = p_logits.shape
    K = K1 - 1
    outcomes, P, Q = _exact_outcomes(p_logits, q_logits)
    total = sum(o[2] for o in outcomes)
    assert abs(total - 1.0) < 1e-9
    tol = 4 * (K + 2) / G
    for j in range(K1):
        reach = {}      # prefix (len j) -> P(n >= j, out[0..j-1] = prefix)
        emit = {}       # prefix + (v,) -> P(n >= j, out[0..j] = ...)
        route_acc = {}  # ... via an accepted draft at j
        route_res = {}  # ... via the residual / bonus draw at j
        for seq, route, pr in outcomes:
            n = len(seq) - 1
            if n < j:
                continue
            key = seq[: j + 1]
            reach[seq[:j]] = reach.get(seq[:j], 0.0) + pr
            emit[key] = emit.get(key, 0.0) + pr
            if n > j:
                route_acc[key] = route_acc.get(key, 0.0) + pr
            else:
                route_res[key] = route_res.get(key, 0.0) + pr
        for prefix, r in reach.items():
            for v in range(V):
                key = prefix + (v,)
                assert abs(emit.get(key, 0.0) - r * P[j, v]) < tol, (j, key)
                if j < K:
                    assert abs(route_acc.get(key, 0.0) - r * min(P[j, v], Q[j, v])) < tol
                    assert abs(route_res.get(key, 0.0) - r * max(0.0, P[j, v] - Q[j, v])) < tol


@pytest.mark.parametrize("V,K,seed,sig", [(5, 3, 0, 1.0), (8, 2, 1, 2.0), (3, 3, 2, 3.0),
                                          (4, 1, 3, 0.5), (6, 2, 4, 0.1)])
def test_bruteforce_lossless(V, K, seed, sig):
    rng = np.random.default_rng(seed)
    p = rng.normal(0, 1.5, size=(K + 1, V))
    q = p[:K] + rng.normal(0, sig, size=(K, V))
    _check_lossless(p, q)


def _softmax_at_temperature_2(logits):
    return _ORIG_SOFTMAX(np.asarray(logits, dtype=np.float64) * 0.5)


def _inverse_cdf_off_by_one(weights, u):
    idx, c_prev, c_at, t, tot = _ORIG_INVCDF(weights, u)
    return np.maximum(idx - 1, 0), c_prev, c_at, t, tot


_ORIG_SOFTMAX = oracle_mod.softmax_rows
_ORIG_INVCDF = oracle_mod._inverse_cdf


@pytest.mark.parametrize("name,mutant", [("softmax_rows", _softmax_at_temperature_2),
                                         ("_inverse_cdf", _inverse_cdf_off_by_one)])
def test_bruteforce_catches_planted_oracle_mistakes(monkeypatch, name, mutant):
    """A mistake planted in the oracle (on the CPU) fails the brute-force pin."""
    monkeypatch.setattr(oracle_mod, name, mutant)
    rng = np.random.default_rng(0)
    p = rng.normal(0, 1.5, size=(3, 4))
    q = p[:2] + rng.normal(0, 1.0, size=(2, 4))
    with pytest.raises(AssertionError):
        _check_lossless(p, q)


def test_bruteforce_lossless_with_identical_row_and_masked_tokens():
    rng = np.random.default_rng(9)
    V, K = 5, 3
    p = rng.normal(0, 1.0, size=(K + 1, V))
    q = p[:K] + rng.normal(0, 1.0, size=(K, V))
    q[1] = p[1]                 # position 1: draft equals verifier
    p[2, 0] = -np.inf           # a token the verifier forbids
    q[0, 3] = -np.inf           # a token the draft never proposes
    _check_lossless(p, q)


# --------------------------------------------------------------------------
# statistics with Philox uniforms
# --------------------------------------------------------------------------


def _emitted_stats(p, q, steps, B, seed):
    K = q.shape[0]
    V = p.shape[1]
    firsts = []
    at_j = [[] for _ in range(K + 1)]
    ns = []
    rng = np.random.default_rng(seed + 1000)
    Q = _lib_softmax(q)
    for step in range(steps):
        pb = np.broadcast_to(p, (B,) + p.shape)
        qb = np.broadcast_to(q, (B,) + q.shape)
        x = np.stack([rng.choice(V, size=B, p=Q[i]) for i in range(K)], axis=1)
        res = verify_block(pb, qb, x, seed=seed, step=step)
        out, n = res["out_tokens"], res["accepted_len"]
        firsts.append(out[:, 0])
        for j in range(K + 1):
            at_j[j].append(out[n >= j, j])
        ns.append(n)
    return (np.concatenate(firsts), [np.concatenate(a) for a in at_j], np.concatenate(ns))


def test_chisquare_one_million_draws():
    V, K = 8, 3
    rng = np.random.default_rng(42)
    p = rng.normal(0, 1.2, size=(K + 1, V))
    q = p[:K] + rng.normal(0, 1.0, size=(K, V))
    P = _lib_softmax(p)
    first, at_j, _ = _emitted_stats(p, q, steps=8, B=1 << 17, seed=2024)
    assert first.size == 1 << 20
    counts = np.bincount(first, minlength=V)
    assert stats.chisquare(counts, P[0] * counts.sum()).pvalue > 1e-3
    for j in range(K + 1):
        counts = np.bincount(at_j[j], minlength=V)
        assert counts.sum() > 10_000
        assert stats.chisquare(counts, P[j] * counts.sum()).pvalue > 1e-3


def test_mean_accepted_length_matches_tv():
    V, K, B = 64, 8, 1 << 15
    rng = np.random.default_rng(7)
    p = rng.normal(0, 2.0, size=(K + 1, V))
    q = p[:K] + rng.normal(0, 0.6, size=(K, V))
    P, Q = _lib_softmax(p), _lib_softmax(q)
    tv = 0.5 * np.abs(P[:K] - Q).sum(axis=1)
    expect = sum(np.prod(1 - tv[:j]) for j in range(1, K + 1))
    _, _, n = _emitted_stats(p, q, steps=1, B=B, seed=11)
    assert abs(n.mean() - expect) < 4 * n.std() / np.sqrt(n.size)
    # TPF bound of the pages, in this API's terms: 1 <= n + 1 <= K + 1.
    assert n.min() >= 0 and n.max() <= K


# --------------------------------------------------------------------------
# hand-worked and special cases
# --------------------------------------------------------------------------


def test_golden_k1_v2():
    with open(os.path.join(GOLDEN, "verify_k1_v2.json")) as f:
        g = json.load(f)
    p = np.array(g["p_logits"])[None]
    q = np.array(g["q_logits"])[None]
    for case in g["cases"]:
        res = oracle_mod.verify_block_u(p, q, np.array([[case["draft"]]]),
                             np.array([[case["u_acc"]]]), np.array([case["u_smp"]]))
        assert res["out_tokens"][0].tolist() == case["out"], case["name"]
        assert res["accepted_len"][0] == case["n"], case["name"]


def test_identical_draft_accepts_everything():
    rng = np.random.default_rng(3)
    B, K, V = 64, 8, 100
    p = rng.normal(0, 2, size=(B, K + 1, V))
    x = rng.integers(0, V, size=(B, K))
    res = verify_block(p, p[:, :K], x, seed=5, step=0)
    assert np.all(res["accepted_len"] == K)
    assert np.array_equal(res["out_tokens"][:, :K], x)


def test_concentrated_verifier_rejects_first_and_emits_its_token():
    B, K, V = 32, 4, 50
    rng = np.random.default_rng(4)
    t = rng.integers(0, V, size=B)
    p = np.zeros((B, K + 1, V))
    p[np.arange(B), 0, t] = 200.0
    q = rng.normal(0, 1, size=(B, K, V))
    x = (t[:, None] + 1 + rng.integers(0, V - 1, size=(B, K))) % V
    u_acc, _ = uniforms_for_block(B, K, seed=8, step=3)
    assert np.all(u_acc[:, 0] > 0)  # u = 0 would accept anything with p > 0
    res = verify_block(p, q, x, seed=8, step=3)
    assert np.all(res["accepted_len"] == 0)
    assert np.array_equal(res["out_tokens"][:, 0], t)
    assert np.all(res["out_tokens"][:, 1:] == -1)


def test_disjoint_supports_reject_and_resample_from_p():
    B, K, V = 4096, 2, 10
    p = np.full((B, K + 1, V), -np.inf)
    q = np.full((B, K, V), -np.inf)
    p[:, :, :5] = np.log(np.arange(1, 6))      # p_0 = (1..5)/15 on tokens 0..4
    q[:, :, 5:] = 0.0                            # q uniform on tokens 5..9
    x = np.random.default_rng(0).integers(5, 10, size=(B, K))
    res = verify_block(p, q, x, seed=1, step=0)
    assert np.all(res["accepted_len"] == 0)
    y = res["out_tokens"][:, 0]
    assert y.max() < 5
    assert stats.chisquare(np.bincount(y, minlength=5),
                           np.arange(1, 6) / 15 * B).pvalue > 1e-3


def test_invalid_draft_marks_sequence():
    B, K, V = 4, 3, 16
    rng = np.random.default_rng(1)
    p = rng.normal(size=(B, K + 1, V))
    q = rng.normal(size=(B, K, V))
    x = rng.integers(0, V, size=(B, K))
    x[1, 2] = V
    x[3, 0] = -1
    res = verify_block(p, q, x, seed=0, step=0)
    assert res["accepted_len"][1] == -1 and res["accepted_len"][3] == -1
    assert np.all(res["out_tokens"][[1, 3]] == -1)
    # Sequence b draws from counter b, so row 0 matches a call holding row 0 alone.
    alone = verify_block(p[:1], q[:1], x[:1], seed=0, step=0)
    assert alone["accepted_len"][0] == res["accepted_len"][0] >= 0
    assert np.array_equal(alone["out_tokens"][0], res["out_tokens"][0])


def test_empty_residual_falls_back_to_p():
    K, V = 2, 6
    rng = np.random.default_rng(2)
    p = rng.normal(size=(1, K + 1, V))
    q = p[:, :K].copy()
    x = np.array([[1, 2]])
    # u = 1 lies outside [0, 1); it forces a rejection where p = q.
    res = oracle_mod.verify_block_u(p, q, x, np.array([[1.0, 0.0]]), np.array([[0.5, 0.0, 0.0]]))
    assert res["accepted_len"][0] == 0
    P = _lib_softmax(p[0, 0])
    cdf = np.cumsum(P)
    assert res["out_tokens"][0, 0] == int(np.argmax(cdf > 0.5 * cdf[-1]))


def test_row_statistics_match_library():
    rng = np.random.default_rng(6)
    B, K, V = 3, 4, 257
    p = rng.normal(0, 3, size=(B, K + 1, V))
    q = rng.normal(0, 3, size=(B, K, V))
    x = rng.integers(0, V, size=(B, K))
    res = verify_block(p, q, x, seed=1, step=2)
    lse = np.concatenate([special.logsumexp(p, axis=-1), special.logsumexp(q, axis=-1)], axis=1)
    assert np.allclose(res["row_lse"], lse, rtol=0, atol=1e-12)
    P, Q = _lib_softmax(p), _lib_softmax(q)
    assert np.allclose(res["p_at_draft"], np.take_along_axis(P[:, :K], x[..., None], 2)[..., 0],
                       atol=1e-15)
    assert np.allclose(res["q_at_draft"], np.take_along_axis(Q, x[..., None], 2)[..., 0],
                       atol=1e-15)


def test_softmax_hand_values_and_invariants():
    probs, lse = softmax_rows(np.array([[0.0, np.log(3.0)], [0.0, 0.0], [5.0, -np.inf]]))
    assert np.allclose(probs[0], [0.25, 0.75], atol=1e-15)
    assert np.allclose(probs[1], [0.5, 0.5], atol=0)
    assert probs[2].tolist() == [1.0, 0.0]
    assert abs(lse[1] - np.log(2.0)) < 1e-15
    rng = np.random.default_rng(0)
    l = rng.normal(0, 10, size=(8, 1000))
    pr, _ = softmax_rows(l)
    assert np.all(np.abs(pr.sum(axis=1) - 1) < 1e-12)
    pr2, _ = softmax_rows(l + 123.25)
    assert np.allclose(pr, pr2, rtol=1e-12, atol=0)
