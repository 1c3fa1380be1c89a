"""Pins of the oracle's tree sampler (top-k candidates per position, the kept
sequences, the prefix tree and its lossless walk).

Pages: "Unlocking Lossless Speedups in LLMs via Discrete Diffusion" --
paperglide reader, The Psi-Speculative Sampler (worked example with
(B, K, V) = (3, 2, 2): K^(B-1) candidates ranked by joint log-probability,
the top V prefixes kept and verified by the AR model) and Sampler Extensions;
picx.dev summary, Methodology / Psi-Speculative Sampler (tree sampler: top-K
at each position). The pins never compare the oracle with itself:

* hand-worked trees and walks (tests/golden/tree_hand.json);
* the kept set: the oracle's full enumeration (the pages' definition) and
  its best-first search (used when top_k^D is large) agree, with ties, and
  best-first matches a numpy argsort of all 6^6 joint scores;
* closed forms: the best sequence is the per-position argmax, a depth-1 tree
  is the top-budget tokens of q_1, budget = top_k^D keeps every combination;
* invariants: parents precede children, every kept sequence is a root-leaf
  path, shifting a row of logits changes nothing;
* losslessness: the walk's uniforms are integrated exactly over their
  2^24-point grid and the probability of every emitted sequence must equal
  the chain-rule product of the AR rows along its prefix.
"""

import json
import os

import numpy as np
import pytest
from scipy import special

import oracle.tree_sampler as tree_mod
from oracle import (tree_build, tree_candidates, tree_draft, tree_topk, tree_uniforms,
                    tree_verify, tree_verify_u, uniforms_for_block)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
G = 1 << 24


def _log(p):
    p = np.asarray(p, dtype=np.float64)
    with np.errstate(divide="ignore"):
        return np.where(p > 0, np.log(np.where(p > 0, p, 1.0)), -np.inf)


def _golden():
    with open(os.path.join(GOLDEN, "tree_hand.json")) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# hand-worked cases
# --------------------------------------------------------------------------


@pytest.mark.parametrize("case", [c["name"] for c in _golden()["trees"]])
def test_golden_trees(case):
    c = next(t for t in _golden()["trees"] if t["name"] == case)
    q = _log(c["q"])[None]
    tree = tree_draft(q, c["top_k"], c["budget"])
    n = len(c["node_token"])
    assert tree["n_nodes"][0] == n
    assert tree["node_token"][0, :n].tolist() == c["node_token"]
    assert tree["node_parent"][0, :n].tolist() == c["node_parent"]
    assert tree["node_depth"][0, :n].tolist() == c["node_depth"]
    assert (tree["node_token"][0, n:] == -1).all() and (tree["node_depth"][0, n:] == -1).all()
    ids = tree["topk_ids"][0]
    kept = [[int(ids[i, s]) for i, s in enumerate(tup)] for tup, _ in tree["kept"][0]]
    assert kept == c["kept_tokens"]
    probs = [np.exp(score) for _, score in tree["kept"][0]]
    assert np.allclose(probs, c["kept_prob"], rtol=1e-12)


def test_golden_walks():
    g = _golden()
    w = g["walk"]
    c = next(t for t in g["trees"] if t["name"] == w["tree"])
    tree = tree_draft(_log(c["q"])[None], c["top_k"], c["budget"])
    p = _log(w["p"])[None]
    for case in w["cases"]:
        res = tree_verify_u(p, tree["node_token"], tree["node_parent"], tree["n_nodes"],
                            np.array([case["u"]]))
        assert res["out_tokens"][0].tolist() == case["out"], case
        assert res["accepted_len"][0] == case["accepted"], case


# --------------------------------------------------------------------------
# the kept set: an independent best-first enumeration
# --------------------------------------------------------------------------


@pytest.mark.parametrize("seed", range(12))
def test_kept_set_enumeration_equals_best_first_search(seed):
    """The oracle's two routes to the kept set (full enumeration, the pages'
    definition; best-first search, used when top_k^D is large) agree,
    including exact ties and rows with few candidates."""
    rng = np.random.default_rng(seed)
    D, k, budget = int(rng.integers(1, 5)), int(rng.integers(1, 5)), int(rng.integers(1, 12))
    V = 12
    # quantised logits make exact ties in the per-position lists and in the sums
    q = np.round(rng.normal(0, 1.5, size=(1, D, V)) * 2) / 2
    if seed % 3 == 0:
        q[0, 0, rng.integers(0, V, size=V - 2)] = -np.inf  # a row with few candidates
    ids, logq = tree_topk(q, k)
    got = tree_candidates(logq[0], budget, method="enumerate")
    want = tree_candidates(logq[0], budget, method="best_first")
    assert [t for t, _ in got] == [t for t, _ in want]
    assert np.allclose([s for _, s in got], [s for _, s in want], rtol=0, atol=1e-12)


def test_best_first_against_sorted_brute_force_list():
    """Best-first at a size where enumeration is the textbook check: the
    first 50 of 6^6 = 46656 sequences, every joint score recomputed from the
    per-position log-probabilities with numpy broadcasting and argsort."""
    rng = np.random.default_rng(77)
    D, k = 6, 6
    logq = np.sort(rng.normal(-3, 1, size=(D, k)), axis=1)[:, ::-1]
    grids = np.meshgrid(*[np.arange(k)] * D, indexing="ij")
    tup = np.stack([g.reshape(-1) for g in grids], axis=1)
    total = sum(logq[i][tup[:, i]] for i in range(D))
    order = np.lexsort(tuple(tup[:, i] for i in reversed(range(D))) + (-total,))
    want = [tuple(int(x) for x in tup[o]) for o in order[:50]]
    got = [t for t, _ in tree_candidates(logq, 50, method="best_first")]
    assert got == want


def test_topk_order_ties_and_masks():
    q = np.array([[[1.0, 3.0, 3.0, -np.inf, 2.0, 3.0]]])
    ids, logq = tree_topk(q, 4)
    assert ids[0, 0].tolist() == [1, 2, 5, 4]
    lse = np.log(np.exp(1.0) + 3 * np.exp(3.0) + np.exp(2.0))
    assert np.allclose(logq[0, 0], [3 - lse, 3 - lse, 3 - lse, 2 - lse])
    ids, logq = tree_topk(np.array([[[0.0, -np.inf, -np.inf]]]), 3)
    assert ids[0, 0].tolist() == [0, -1, -1] and np.isneginf(logq[0, 0, 1:]).all()


# --------------------------------------------------------------------------
# closed forms and invariants
# --------------------------------------------------------------------------


def test_best_sequence_is_per_position_argmax():
    rng = np.random.default_rng(3)
    q = rng.normal(0, 2, size=(4, 3, 50))
    tree = tree_draft(q, 3, 5)
    for b in range(4):
        tup, score = tree["kept"][b][0]
        assert tup == (0, 0, 0)
        assert [int(tree["topk_ids"][b, i, 0]) for i in range(3)] == q[b].argmax(axis=1).tolist()
        ref = sum(q[b, i].max() - special.logsumexp(q[b, i]) for i in range(3))
        assert abs(score - ref) < 1e-12


def test_depth_one_tree_is_top_budget_of_q1():
    rng = np.random.default_rng(5)
    q = rng.normal(0, 2, size=(3, 1, 40))
    for budget in (1, 3, 6):
        tree = tree_draft(q, 6, budget)
        for b in range(3):
            n = int(tree["n_nodes"][b])
            assert n == 1 + budget
            want = np.argsort(-q[b, 0], kind="stable")[:budget]
            assert tree["node_token"][b, 1:n].tolist() == want.tolist()
            assert (tree["node_parent"][b, 1:n] == 0).all()


def test_full_budget_keeps_every_combination():
    rng = np.random.default_rng(6)
    D, k = 3, 3
    q = rng.normal(0, 1, size=(1, D, 20))
    tree = tree_draft(q, k, k ** D)
    # a complete k-ary tree of depth D
    assert tree["n_nodes"][0] == sum(k ** j for j in range(D + 1))
    for d in range(1, D + 1):
        assert (tree["node_depth"][0] == d).sum() == k ** d


@pytest.mark.parametrize("seed", range(6))
def test_tree_structure_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    B, D, k, budget, V = 3, int(rng.integers(1, 5)), int(rng.integers(1, 4)), int(rng.integers(1, 9)), 30
    q = rng.normal(0, 2, size=(B, D, V))
    tree = tree_draft(q, k, budget)
    for b in range(B):
        n = int(tree["n_nodes"][b])
        tok, par, dep = (tree[f][b] for f in ("node_token", "node_parent", "node_depth"))
        assert dep[0] == 0 and par[0] == -1 and tok[0] == -1
        for c in range(1, n):
            assert 0 <= par[c] < c and dep[c] == dep[par[c]] + 1
        # siblings carry distinct tokens
        for c in range(n):
            kids = [tok[x] for x in range(1, n) if par[x] == c]
            assert len(kids) == len(set(kids))
        # every kept sequence is a root-to-leaf path, and every leaf is one
        paths = set()
        for c in range(1, n):
            if dep[c] == D:
                seq, x = [], c
                while x > 0:
                    seq.append(int(tok[x]))
                    x = par[x]
                paths.add(tuple(reversed(seq)))
        kept = {tuple(int(tree["topk_ids"][b, i, s]) for i, s in enumerate(t))
                for t, _ in tree["kept"][b]}
        assert paths == kept
        assert len(kept) == min(budget, k ** D)


def test_shifting_a_row_changes_nothing():
    rng = np.random.default_rng(8)
    q = rng.normal(0, 2, size=(2, 3, 25))
    t0 = tree_draft(q, 3, 7)
    q2 = q + rng.normal(0, 5, size=(2, 3, 1))
    t1 = tree_draft(q2, 3, 7)
    for f in ("node_token", "node_parent", "node_depth", "n_nodes"):
        assert np.array_equal(t0[f], t1[f])


# --------------------------------------------------------------------------
# losslessness of the walk, by exact integration over the uniform grid
# --------------------------------------------------------------------------


def _exact_walk_distribution(tree, p_logits, b):
    """{emitted tuple: probability} of the oracle's walk of sequence b, every
    depth's uniform integrated exactly over its 2^24-point grid.

    The draw at depth j is monotone in u_j once u_0 .. u_{j-1} are fixed, so
    each token owns one interval of the grid; its ends come from binary
    search on full walks (module attribute, so a planted mistake is seen)
    with the earlier uniforms at representatives of the tokens taken so far.
    """
    tok = tree["node_token"][b:b + 1]
    par = tree["node_parent"][b:b + 1]
    n = tree["n_nodes"][b:b + 1]
    D = tree["topk_ids"].shape[1]
    p = p_logits[b:b + 1]
    dist = {}

    def out_at(us, j):
        u = np.zeros((1, D + 1))
        u[0, :len(us)] = np.asarray(us, dtype=np.float64) * 2.0**-24
        res = tree_mod.tree_verify_u(p, tok, par, n, u)
        return int(res["out_tokens"][0, j]), int(res["accepted_len"][0])

    def rec(us, prefix, prob):
        j = len(us)
        V = p.shape[2]
        lo_g = 0
        for v in range(V):
            lo, hi = lo_g, G
            while lo < hi:  # first g whose draw at depth j exceeds v
                mid = (lo + hi) // 2
                if out_at(us + [mid], j)[0] > v:
                    hi = mid
                else:
                    lo = mid + 1
            cnt, start = lo - lo_g, lo_g
            lo_g = lo
            if cnt == 0:
                continue
            y, acc = out_at(us + [start], j)
            assert y == v
            pr = prob * cnt / G
            if acc > j:  # the walk moved on: the token was a child
                rec(us + [start], prefix + (v,), pr)
            else:
                dist[prefix + (v,)] = dist.get(prefix + (v,), 0.0) + pr

    rec([], (), 1.0)
    return dist


def _check_walk_lossless(tree, p_logits, b):
    """Every emitted sequence has the chain-rule probability of the AR rows
    along its prefix; the node of each prefix is found from the tree's
    tokens, not from the oracle's walk."""
    tok, par, n = tree["node_token"][b], tree["node_parent"][b], int(tree["n_nodes"][b])
    P = special.softmax(p_logits[b], axis=-1)
    dist = _exact_walk_distribution(tree, p_logits, b)
    assert abs(sum(dist.values()) - 1.0) < 1e-9
    D = tree["topk_ids"].shape[1]
    for seq, prob in dist.items():
        node, want = 0, 1.0
        for j, y in enumerate(seq):
            want *= P[node, y]
            if j < len(seq) - 1:
                node = next(c for c in range(1, n) if par[c] == node and tok[c] == y)
        assert abs(prob - want) <= (D + 1) * 2.0**-24, (seq, prob, want)


@pytest.mark.parametrize("seed", range(4))
def test_walk_is_lossless_by_exact_integration(seed):
    rng = np.random.default_rng(200 + seed)
    V, D, k, budget = 4, 2, 2, 3
    q = rng.normal(0, 1, size=(1, D, V))
    tree = tree_draft(q, k, budget)
    N = tree["node_token"].shape[1]
    p = rng.normal(0, 1, size=(1, N, V))
    if seed == 1:
        p[0, :, 3] = -np.inf  # a token the verifier never emits
    if seed == 2:
        p[0, 0] = np.log([0.7, 0.1, 0.1, 0.1])  # q's favourites need not be p's
    _check_walk_lossless(tree, p, 0)


_real_walk = tree_mod.tree_verify_u


def _walk_uses_parent_row(p_logits, node_token, node_parent, n_nodes, u):
    """Planted mistake: below the root, draw from the parent's row."""
    p = np.asarray(p_logits, dtype=np.float64).copy()
    shifted = p.copy()
    for b in range(p.shape[0]):
        for c in range(1, int(n_nodes[b])):
            shifted[b, c] = p[b, node_parent[b, c]]
    return _real_walk(shifted, node_token, node_parent, n_nodes, u)


def _walk_off_by_one_depth_uniform(p_logits, node_token, node_parent, n_nodes, u):
    """Planted mistake: depth j draws with the uniform of depth j - 1."""
    u = np.asarray(u, dtype=np.float64).copy()
    u[:, 1:] = u[:, :-1].copy()
    return _real_walk(p_logits, node_token, node_parent, n_nodes, u)


@pytest.mark.parametrize("mutant", [_walk_uses_parent_row, _walk_off_by_one_depth_uniform])
def test_exact_integration_catches_planted_walk_mistakes(monkeypatch, mutant):
    rng = np.random.default_rng(9)
    q = rng.normal(0, 1, size=(1, 2, 4))
    tree = tree_draft(q, 2, 3)
    p = rng.normal(0, 1.5, size=(1, tree["node_token"].shape[1], 4))
    _check_walk_lossless(tree, p, 0)
    monkeypatch.setattr(tree_mod, "tree_verify_u", mutant)
    with pytest.raises(AssertionError):
        _check_walk_lossless(tree, p, 0)


# --------------------------------------------------------------------------
# uniforms and degenerate cases
# --------------------------------------------------------------------------


def test_tree_uniforms_are_the_sampling_words():
    u = tree_uniforms(3, 5, seed=11, step=7)
    assert u.shape == (3, 6)
    assert np.array_equal(u, uniforms_for_block(3, 5, 11, 7)[1])


def test_walk_monte_carlo_first_token_follows_root_row():
    rng = np.random.default_rng(12)
    V = 6
    q = rng.normal(0, 1, size=(1, 2, V))
    tree = tree_draft(q, 2, 2)
    N = tree["node_token"].shape[1]
    p = rng.normal(0, 1, size=(1, N, V))
    P0 = special.softmax(p[0, 0])
    n_draws = 20000
    pb = np.broadcast_to(p, (n_draws, N, V))
    tb = {f: np.broadcast_to(tree[f], (n_draws,) + tree[f].shape[1:]) for f in
          ("node_token", "node_parent", "n_nodes")}
    res = tree_verify_u(pb, tb["node_token"], tb["node_parent"], tb["n_nodes"],
                        tree_uniforms(n_draws, 2, seed=5, step=0))
    first = res["out_tokens"][:, 0]
    freq = np.bincount(first, minlength=V) / n_draws
    se = np.sqrt(P0 * (1 - P0) / n_draws)
    assert (np.abs(freq - P0) <= 5 * se + 1e-12).all()


def test_invalid_row_on_the_walk_marks_the_sequence():
    g = _golden()
    c = next(t for t in g["trees"] if t["name"] == "branch_at_depth_1")
    tree = tree_draft(_log(c["q"])[None], c["top_k"], c["budget"])
    p = _log(g["walk"]["p"])[None]
    p[0, 1] = -np.inf  # node 1 (prefix [2]) has no distribution
    res = tree_verify_u(p, tree["node_token"], tree["node_parent"], tree["n_nodes"],
                        np.array([[0.5, 0.2, 0.9]]))
    assert res["accepted_len"][0] == -1 and (res["out_tokens"][0] == -1).all()
    # a walk that never reaches node 1 is unaffected
    res = tree_verify_u(p, tree["node_token"], tree["node_parent"], tree["n_nodes"],
                        np.array([[0.1, 0.8, 0.6]]))
    assert res["out_tokens"][0].tolist() == [0, 1, 1]


def test_empty_candidates_give_a_root_only_tree():
    q = np.full((1, 2, 5), -np.inf)
    q[0, 0, 1] = 0.0  # position 2 has no finite logit: no candidate sequence
    tree = tree_draft(q, 2, 4)
    assert tree["n_nodes"][0] == 1
    p = np.zeros((1, tree["node_token"].shape[1], 5))
    res = tree_verify(p, tree, seed=1, step=0)
    assert res["accepted_len"][0] == 0 and res["out_tokens"][0, 0] >= 0
    assert (res["out_tokens"][0, 1:] == -1).all()


def test_build_accepts_precomputed_topk():
    rng = np.random.default_rng(13)
    q = rng.normal(0, 1, size=(2, 3, 16))
    ids, logq = tree_topk(q, 3)
    a = tree_build(ids, logq, 5)
    b = tree_draft(q, 3, 5)
    for f in ("node_token", "node_parent", "node_depth", "n_nodes"):
        assert np.array_equal(a[f], b[f])


def test_walk_draws_at_every_node_follow_its_row():
    """Monte Carlo over Philox uniforms: among walks that reach a node, the
    token drawn there is distributed as softmax of that node's AR row
    (chi-square per node), so each depth's uniform is independent of the
    path and the walk reads the right row."""
    from scipy import stats as st
    rng = np.random.default_rng(21)
    V, D = 5, 2
    q = rng.normal(0, 1, size=(1, D, V))
    tree = tree_draft(q, 2, 3)
    N = tree["node_token"].shape[1]
    p = rng.normal(0, 0.8, size=(1, N, V))
    for c in range(1, int(tree["n_nodes"][0])):  # make the tree's tokens likely
        p[0, tree["node_parent"][0, c], tree["node_token"][0, c]] += 1.5
    n_draws = 40000
    pb = np.broadcast_to(p, (n_draws, N, V))
    tb = {f: np.broadcast_to(tree[f], (n_draws,) + tree[f].shape[1:]) for f in
          ("node_token", "node_parent", "n_nodes")}
    res = tree_verify_u(pb, tb["node_token"], tb["node_parent"], tb["n_nodes"],
                        tree_uniforms(n_draws, D, seed=17, step=4))
    out = res["out_tokens"]
    tok, par = tree["node_token"][0], tree["node_parent"][0]
    P = special.softmax(p[0], axis=-1)
    # node reached by each walk at each depth, found from the emitted tokens
    node = np.zeros(n_draws, dtype=np.int64)
    checked = 0
    for j in range(D + 1):
        live = out[:, j] >= 0
        for n in np.unique(node[live]):
            sel = live & (node == n)
            if sel.sum() < 500:
                continue
            counts = np.bincount(out[sel, j], minlength=V)
            assert st.chisquare(counts, P[n] * sel.sum()).pvalue > 1e-4, (j, n)
            checked += 1
        # advance along accepted tokens
        nxt = np.full(n_draws, -1)
        for c in range(1, int(tree["n_nodes"][0])):
            hit = live & (par[c] == node) & (out[:, j] == tok[c]) & (res["accepted_len"] > j)
            nxt[hit] = c
        node = np.where(nxt >= 0, nxt, node)  # stopped walks are -1 from here on
    assert checked >= 3
