"""Parity of the CUDA tree sampler with the float64 oracle, on a B200.

* top-k: ids bit-exact (the decision is on the logits as stored, exact on
  both sides), log-probabilities within 2e-5;
* the tree: node arrays bit-exact, except sequences whose budget boundary is
  a near tie (the budget-th and the next best joint log-probability within
  1e-4 in the oracle; the device sums float32): those are counted and checked
  to be a valid answer (canonical node order, as many leaves as the oracle
  keeps, each within the tie band of the oracle's last kept score);
* the walk, on the oracle's tree: every node's draw equals the oracle's
  inverse-CDF draw with the same uniform except near ties of the draw rule;
  emitted tokens and accepted lengths equal the oracle's for sequences with
  no near-tie draw on their path.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_decoding_b200.inputs import verify_inputs
from tests.parity import TAU_DRAFT, widen

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SCORE_TIE = 1e-4


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_decoding_b200 import api as A
    return A


def _q(B, D, V, dtype, dist="normal", seed=0):
    return verify_inputs(B, D, V, dtype=dtype, dist=dist, seed=seed, device=DEV).q_logits


def _p(B, N, V, dtype, seed=0):
    return verify_inputs(B, N - 1, V, dtype=dtype, dist="normal", seed=seed + 7,
                         device=DEV).p_logits


def _check_topk(tree, qw, top_k):
    ids, logq = oracle.tree_topk(qw, top_k)
    got_i = tree.topk_ids.cpu().numpy()
    got_l = tree.topk_logq.cpu().numpy().astype(np.float64)
    assert np.array_equal(got_i, ids)
    fin = ids >= 0
    assert np.all(np.isneginf(got_l[~fin]))
    assert np.abs(got_l[fin] - logq[fin]).max(initial=0.0) < 2e-5
    return ids, logq


def _check_valid_tree(tree, b, ids_b, logq_b, kept):
    """A tree whose budget boundary is a near tie: not unique, so check that
    it is a valid answer. Nodes in canonical order (depth, then rank tuple),
    parents before children, and as many leaves as the oracle keeps, each a
    sequence whose oracle score is within SCORE_TIE of the oracle's last
    kept one."""
    n = int(tree.n_nodes[b])
    tok = tree.node_token[b].cpu().numpy()
    par = tree.node_parent[b].cpu().numpy()
    dep = tree.node_depth[b].cpu().numpy()
    D = ids_b.shape[0]
    assert dep[0] == 0 and par[0] == -1 and (tok[n:] == -1).all() and (dep[n:] == -1).all()
    rank_of = [{int(v): s for s, v in enumerate(ids_b[i]) if v >= 0} for i in range(D)]
    tuples = [()]
    for c in range(1, n):
        assert 0 <= par[c] < c and dep[c] == dep[par[c]] + 1
        tuples.append(tuples[par[c]] + (rank_of[dep[c] - 1][int(tok[c])],))
    keys = [(len(t), t) for t in tuples[1:]]
    assert keys == sorted(keys) and len(set(keys)) == len(keys)
    leaves = [t for t in tuples if len(t) == D]
    assert len(leaves) == len(kept)
    last = kept[-1][1]
    for t in leaves:
        score = sum(logq_b[i, s] for i, s in enumerate(t))
        assert score >= last - SCORE_TIE, (t, score, last)


def _check_tree(tree, ids, logq, budget):
    """Node arrays against the oracle's tree; returns (compared, ties)."""
    ref = oracle.tree_build(ids, logq, budget)
    B = ids.shape[0]
    compared = ties = 0
    for b in range(B):
        nxt = oracle.tree_candidates(logq[b], budget + 1)
        if len(nxt) > budget and nxt[budget - 1][1] - nxt[budget][1] < SCORE_TIE:
            _check_valid_tree(tree, b, ids[b], logq[b], ref["kept"][b])
            ties += 1
            continue
        for f in ("node_token", "node_parent", "node_depth"):
            got = getattr(tree, f)[b].cpu().numpy()
            assert np.array_equal(got, ref[f][b]), (f, b, got, ref[f][b])
        assert int(tree.n_nodes[b]) == ref["n_nodes"][b]
        compared += 1
    return compared, ties


@pytest.mark.parametrize("B,D,V,dtype,top_k,budget,dist", [
    (2, 3, 1000, "f32", 2, 2, "normal"),      # the pages' shape (3, 2, 2) over D = 2 .. 3
    (3, 1, 4097, "bf16", 5, 3, "gumbel"),     # depth 1, odd V (unaligned rows)
    (4, 15, 32000, "bf16", 4, 16, "normal"),
    (2, 16, 2048, "f32", 16, 64, "normal"),   # largest depth, top_k, budget
    (5, 7, 3000, "bf16", 10, 60, "gumbel"),   # depth 7, top-10, budget 60
    (1, 4, 5, "f32", 8, 20, "normal"),        # V below top_k: missing slots
])
def test_draft_parity(api, B, D, V, dtype, top_k, budget, dist):
    q = _q(B, D, V, dtype, dist, seed=V + D)
    tree = api.tree_draft(q, top_k, budget)
    torch.cuda.synchronize()
    ids, logq = _check_topk(tree, widen(q), top_k)
    compared, ties = _check_tree(tree, ids, logq, budget)
    assert compared + ties == B


def test_draft_ties_and_masks(api):
    g = torch.Generator().manual_seed(5)
    q = (torch.randn(4, 5, 600, generator=g) * 2).round() / 2  # exact ties everywhere
    q[0, 2, :590] = float("-inf")       # ten candidates left
    q[1, 1, :] = float("-inf")          # none: root-only tree
    q[2, 0, :599] = float("-inf")       # one
    qd = q.to(DEV)
    tree = api.tree_draft(qd, 6, 12)
    torch.cuda.synchronize()
    ids, logq = _check_topk(tree, q.double().numpy(), 6)
    compared, ties = _check_tree(tree, ids, logq, 12)
    assert compared + ties == 4
    assert int(tree.n_nodes[1]) == 1


def _oracle_tree_on_device(ref):
    return {f: torch.as_tensor(ref[f], dtype=torch.int32, device=DEV)
            for f in ("node_token", "node_parent", "node_depth", "n_nodes")}


def _check_walk(api, ref, p, seed, step, D, budget):
    """Device walk on the oracle's tree; returns (sequences compared, ties)."""
    t = _oracle_tree_on_device(ref)
    tree = api.DraftTree(ref["topk_ids_t"], ref["topk_logq_t"], t["node_token"],
                         t["node_parent"], t["node_depth"], t["n_nodes"], budget)
    res = api.tree_verify(p, tree, seed, step)
    torch.cuda.synchronize()
    pw = widen(p)
    B, N, V = pw.shape
    u = oracle.tree_uniforms(B, D, seed, step)
    draw = res.node_draw.cpu().numpy()
    ties_at = np.zeros((B, N), dtype=bool)
    for b in range(B):
        n = int(ref["n_nodes"][b])
        assert (draw[b, n:] == -1).all()
        for c in range(n):
            j = int(ref["node_depth"][b, c])
            ids, det = oracle.sample_drafts_u(pw[b, c][None, None], u[b, j][None, None])
            tie = (min(det["threshold"] - det["c_prev"], det["c_at"] - det["threshold"])
                   < TAU_DRAFT * det["spread"]).item() and ids[0, 0] >= 0
            ties_at[b, c] = tie
            if not tie:
                assert draw[b, c] == ids[0, 0], (b, c, draw[b, c], ids[0, 0])
    want = oracle.tree_verify_u(pw, ref["node_token"], ref["node_parent"], ref["n_nodes"], u)
    out = res.out_tokens.cpu().numpy()
    acc = res.accepted_len.cpu().numpy()
    compared = ties = 0
    for b in range(B):
        # the oracle's path: node of each emitted prefix
        node, on_path = 0, [0]
        for y in want["out_tokens"][b][:max(int(want["accepted_len"][b]), 0)]:
            node = next(c for c in range(1, int(ref["n_nodes"][b]))
                        if ref["node_parent"][b, c] == node and ref["node_token"][b, c] == y)
            on_path.append(node)
        if ties_at[b, on_path].any():
            ties += 1
            continue
        assert np.array_equal(out[b], want["out_tokens"][b]), (b, out[b], want["out_tokens"][b])
        assert acc[b] == want["accepted_len"][b]
        compared += 1
    return compared, ties


def _ref_tree(q, top_k, budget):
    ref = oracle.tree_draft(widen(q), top_k, budget)
    ref["topk_ids_t"] = torch.as_tensor(ref["topk_ids"], dtype=torch.int32, device=DEV)
    ref["topk_logq_t"] = torch.as_tensor(ref["topk_logq"], dtype=torch.float32, device=DEV)
    return ref


@pytest.mark.parametrize("B,D,V,dtype,top_k,budget", [
    (3, 2, 1000, "f32", 2, 2),
    (4, 6, 4097, "bf16", 3, 10),
    (2, 15, 32000, "bf16", 4, 16),
    (2, 16, 3000, "f32", 16, 64),
])
def test_walk_parity(api, B, D, V, dtype, top_k, budget):
    q = _q(B, D, V, dtype, seed=D)
    ref = _ref_tree(q, top_k, budget)
    N = oracle.tree_max_nodes(D, budget)
    # verifier rows built to agree with the tree: each node's row puts its
    # children among the likely tokens, so walks go deep
    p = _p(B, N, V, dtype, seed=V)
    pf = p.float()
    for b in range(B):
        for c in range(1, int(ref["n_nodes"][b])):
            par = int(ref["node_parent"][b, c])
            pf[b, par, int(ref["node_token"][b, c])] += 14.0
    p = pf.to(p.dtype)
    for seed, step in ((1, 0), (77, 31)):
        compared, ties = _check_walk(api, ref, p, seed, step, D, budget)
        assert compared + ties == B and compared >= B - 1


def test_walk_invalid_rows_and_unused_rows(api):
    B, D, V, budget = 3, 3, 500, 4
    q = _q(B, D, V, "f32", seed=11)
    ref = _ref_tree(q, 2, budget)
    N = oracle.tree_max_nodes(D, budget)
    p = _p(B, N, V, "f32", seed=12)
    p[1, 0, :] = float("-inf")  # sequence 1: the root has no distribution
    t = _oracle_tree_on_device(ref)
    tree = api.DraftTree(ref["topk_ids_t"], ref["topk_logq_t"], t["node_token"],
                         t["node_parent"], t["node_depth"], t["n_nodes"], budget)
    res = api.tree_verify(p, tree, 3, 4)
    torch.cuda.synchronize()
    assert int(res.accepted_len[1]) == -1 and (res.out_tokens[1] == -1).all()
    want = oracle.tree_verify_u(widen(p), ref["node_token"], ref["node_parent"], ref["n_nodes"],
                                oracle.tree_uniforms(B, D, 3, 4))
    assert want["accepted_len"][1] == -1
    for b in range(B):
        n = int(ref["n_nodes"][b])
        assert (res.node_draw[b, n:] == -1).all()


def test_end_to_end_qwen3_vocabulary(api):
    """Device draft then device verify at V = 151936 (block of 16: D = 15),
    top-4, budget 16, against the oracle pipeline."""
    B, D, V, top_k, budget = 2, 15, 151936, 4, 16
    q = _q(B, D, V, "bf16", seed=21)
    tree = api.tree_draft(q, top_k, budget)
    torch.cuda.synchronize()
    ids, logq = _check_topk(tree, widen(q), top_k)
    compared, ties = _check_tree(tree, ids, logq, budget)
    assert compared + ties == B
    N = oracle.tree_max_nodes(D, budget)
    p = _p(B, N, V, "bf16", seed=22)
    res = api.tree_verify(p, tree, 9, 2)
    torch.cuda.synchronize()
    ref = _ref_tree(q, top_k, budget)
    c2, t2 = _check_walk(api, ref, p, 9, 2, D, budget)
    assert c2 + t2 == B
    # the device-built tree gives the same walk as the oracle's tree
    if compared == B:
        res2 = api.tree_verify(p, tree, 9, 2)
        torch.cuda.synchronize()
        assert torch.equal(res.out_tokens, res2.out_tokens)
    assert api.device_fault_flags() == 0
