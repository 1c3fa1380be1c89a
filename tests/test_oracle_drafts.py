"""Pins for the oracle's draft sampler (linear sampler proposal): each drafted
id is drawn from softmax(q) of its position by the inverse CDF, with uniforms
from word 2 of the Philox block of that position.

Checked against: a chi-square test of 10^6 draws against scipy's softmax
(not the oracle's), a brute-force CDF written out on tiny rows, -inf masks,
independence of the draft word from the accept and draw words, and the
edge cases (V = 1, a row with no finite logit).
"""
import numpy as np
from scipy.special import softmax as sp_softmax
from scipy.stats import chisquare

from oracle import (draft_uniforms, philox4x32_10, sample_drafts, sample_drafts_u,
                    uniforms_for_block, word_to_uniform)


def test_draws_follow_softmax_chi_square():
    rng = np.random.default_rng(1)
    V, n = 12, 1_000_000
    q = rng.standard_normal(V) * 1.5
    B = n // 2
    logits = np.broadcast_to(q, (B, 2, V))
    ids, _ = sample_drafts(logits, seed=77, step=5)
    counts = np.bincount(ids.reshape(-1), minlength=V)
    expected = sp_softmax(q) * ids.size
    assert chisquare(counts, expected).pvalue > 1e-4


def test_inverse_cdf_by_brute_force():
    rng = np.random.default_rng(2)
    B, K, V = 5, 3, 7
    q = rng.standard_normal((B, K, V))
    u = rng.random((B, K))
    ids, det = sample_drafts_u(q, u)
    for b in range(B):
        for i in range(K):
            w = [np.exp(q[b, i, v] - q[b, i].max()) for v in range(V)]
            total = sum(w)
            run = 0.0
            for v in range(V):
                run += w[v]
                if run > u[b, i] * total:
                    break
            assert ids[b, i] == v
            assert det["c_prev"][b, i] <= det["threshold"][b, i] < det["c_at"][b, i]


def test_masked_tokens_are_never_drafted_and_edge_rows():
    rng = np.random.default_rng(3)
    B, K, V = 64, 4, 9
    q = rng.standard_normal((B, K, V))
    q[..., :4] = -np.inf
    ids, _ = sample_drafts(q, seed=1, step=2)
    assert np.all(ids >= 4)
    one = sample_drafts(np.zeros((3, 2, 1)), seed=4, step=0)[0]
    assert np.all(one == 0)
    dead = np.full((1, 2, 5), -np.inf)
    assert np.all(sample_drafts(dead, seed=4, step=0)[0] == -1)


def test_draft_word_is_word_two_of_the_verifier_block():
    B, K, seed, step = 3, 5, 0x1234_5678_9ABC, 9
    u = draft_uniforms(B, K, seed, step)
    ctr = np.array([[1, 2, step & 0xFFFFFFFF, step >> 32]], dtype=np.uint32)
    key = np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint32)
    assert u[1, 2] == word_to_uniform(philox4x32_10(ctr, key)[0, 2])
    u_acc, u_smp = uniforms_for_block(B, K, seed, step)
    assert not np.any(u == u_acc) and not np.any(u == u_smp[:, :K])
    assert not np.array_equal(u, draft_uniforms(B, K, seed, step + 1))
