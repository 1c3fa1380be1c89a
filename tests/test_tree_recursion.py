"""The device builds the tree sampler's kept set one position at a time:
the best `budget` sequences of j+1 positions extend the best `budget` of j
positions, and a candidate (prefix of rank p, choice of rank s) is considered
only if (p+1)(s+1) <= budget, because every (p' <= p, s' <= s) ranks ahead
of it. This test restates that recursion in Python (float64, so only the
algorithm is under test) and checks it against the oracle's full enumeration
of all top_k^D sequences (the pages' definition), with exact ties, rows with
few candidates and budgets larger than the number of sequences.
"""
import numpy as np
import pytest

from oracle import tree_candidates, tree_topk


def _recursion(logq_b, budget):
    D, k = logq_b.shape
    kept = [((), 0.0)]
    for j in range(D):
        avail = int(np.isfinite(logq_b[j]).sum())
        cand = []
        for p, (tup, score) in enumerate(kept):
            for s in range(min(avail, budget // (p + 1))):
                cand.append((tup + (s,), score + logq_b[j, s]))
        cand.sort(key=lambda c: (-c[1], c[0]))
        kept = cand[:budget]
    return kept


@pytest.mark.parametrize("seed", range(40))
def test_pruned_recursion_equals_full_enumeration(seed):
    rng = np.random.default_rng(1000 + seed)
    D = int(rng.integers(1, 6))
    k = int(rng.integers(1, 7))
    budget = int(rng.integers(1, 50))
    V = 24
    q = rng.normal(0, 1.5, size=(1, D, V))
    if seed % 3 == 0:
        q = np.round(q * 2) / 2  # exact ties within rows and between sums
    if seed % 4 == 1:
        q[0, rng.integers(0, D), rng.integers(0, V, size=V - 2)] = -np.inf
    _, logq = tree_topk(q, k)
    want = tree_candidates(logq[0], budget, method="enumerate")
    got = _recursion(logq[0], budget)
    assert [t for t, _ in got] == [t for t, _ in want]
    assert np.allclose([s for _, s in got], [s for _, s in want], rtol=0, atol=1e-12)


def test_candidate_bound_fits_the_kernel_table():
    """At most 211 candidates per position at budget 64, top-k 16 (the
    kernel's table holds 256)."""
    worst = max(sum(min(k, b // (p + 1)) for p in range(b))
                for b in range(1, 65) for k in range(1, 17))
    assert worst == 211
