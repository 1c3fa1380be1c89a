"""Float64 CPU oracle of the tree variant of the Psi-Spec sampler.

TEST INFRASTRUCTURE, like ``uno_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it; it imports nothing from the CUDA package.

Sources (pages on "Unlocking Lossless Speedups in LLMs via Discrete
Diffusion", Uno):

* [SUM]    picx.dev summary page, "Methodology / Psi-Speculative Sampler":
           the tree sampler draws several candidates by tree-based selection,
           the top K tokens at each position.
* [READER] paperglide reader page, "The Psi-Speculative Sampler" (worked
           example with (B, K, V) = (3, 2, 2): K^(B-1) = 4 candidate
           sequences ranked by joint log-probability, the top V prefixes
           kept, each prefix verified by the AR model, the longest valid one
           accepted) and "Sampler Extensions" (the tree sampler trades
           drafting against verification through (B, K, V)).

The pages' (B, K, V) are the block length, the tokens kept per position and
the verification budget. Here they are ``depth`` D = B - 1 (the positions
after the block's first token, whose logits come from the AR weights alone
and which the linear sampler draws exactly), ``top_k`` and ``budget``; V
remains the vocabulary size.

Readings this module fixes (each also listed in the design notes):

T1. Candidates per position: the top_k ids of the draft logits q_i, ranked by
    logit, larger first, ties to the smaller id. A token whose logit is -inf
    has probability 0 and is never a candidate, so a row with m < top_k
    finite logits offers m candidates (slots beyond them hold id -1).
T2. Joint log-probability of a candidate sequence = sum over positions of
    log softmax(q_i)(x_i): the linear proposal factorises over positions, so
    the joint of the single diffusion pass is the product of its marginals.
T3. The kept set: the ``budget`` sequences of highest joint log-probability
    among all top_k^D, ties broken by the per-position rank tuple in
    lexicographic order (smaller first). Fewer exist only if rows offer fewer
    than top_k candidates.
T4. The tree: node 0 is the root (the state after the block's first token);
    every distinct prefix of a kept sequence is one node. Nodes are ordered
    by depth, then by the rank tuple of their prefix (lexicographic), so a
    parent always precedes its children. The caller's AR pass supplies one
    logit row per node: the AR distribution of the next token after that
    node's prefix.
T5. Lossless verification of a deterministic candidate tree: at the current
    node draw y from the AR distribution of that node (inverse CDF, reading
    4 of the linear oracle, with the sampling uniform of depth j: word 1 of
    the Philox block of (b, j, step)); if y is the token of a child, accept
    it and move there; otherwise emit y and stop. At a leaf the draw is the
    bonus token. Every emitted token is then an exact draw of the AR
    distribution given the tokens before it, which is what "verify each
    prefix with the frozen AR model, keep the longest prefix accepted"
    requires of a lossless sampler.
T6. A node row on the walk with no finite logit marks the sequence invalid:
    accepted length -1 and all output tokens -1.
"""

from __future__ import annotations

import heapq
import itertools

import numpy as np

from .uno_oracle import _inverse_cdf, uniforms_for_block


def tree_topk(q_logits, top_k: int):
    """Per (sequence, position) the top_k candidates (reading T1) and their
    log-probabilities log softmax(q_i) (reading T2).

    q_logits [B, D, V]. Returns (ids [B, D, top_k] int32, logq [B, D, top_k]
    float64); unused slots hold id -1 and logq -inf.
    """
    q = np.asarray(q_logits, dtype=np.float64)
    B, D, V = q.shape
    ids = np.full((B, D, top_k), -1, dtype=np.int32)
    logq = np.full((B, D, top_k), -np.inf)
    for b in range(B):
        for i in range(D):
            row = q[b, i]
            fin = np.isfinite(row)
            if not fin.any():
                continue
            m = row[fin].max()
            lse = m + np.log(np.sum(np.exp(row[fin] - m)))
            cand = np.flatnonzero(fin)
            # sort by logit (larger first), then by id (smaller first)
            order = cand[np.lexsort((cand, -row[cand]))]
            for s, v in enumerate(order[:top_k]):
                ids[b, i, s] = v
                logq[b, i, s] = row[v] - lse
    return ids, logq


ENUMERATE_LIMIT = 200_000  # combinations enumerated outright, at most


def tree_candidates(logq_b, budget: int, method: str = "auto"):
    """The kept sequences of one sequence's block (reading T3).

    logq_b [D, top_k] (slots with -inf are absent). The pages' definition:
    enumerate every combination of one candidate per position, rank them by
    joint log-probability (larger first; ties by rank tuple, smaller first)
    and keep ``budget`` ("enumerate"). When there are more than
    ENUMERATE_LIMIT combinations (top_k^D grows fast) the same total order is
    walked best first ("best_first"): the successors of a rank tuple raise one
    coordinate at or after its last raised one, so every tuple has exactly one
    predecessor, which precedes it in the order (the per-position lists are
    sorted, so its score is not smaller, and on equal scores its tuple is
    smaller). "auto" picks by the count. Returns a list of (rank tuple, joint
    log-probability) in rank order.
    """
    logq_b = np.asarray(logq_b, dtype=np.float64)
    D, k = logq_b.shape
    per_pos = [[s for s in range(k) if np.isfinite(logq_b[i, s])] for i in range(D)]

    def score(tup):
        return float(sum(logq_b[i, s] for i, s in enumerate(tup)))

    count = int(np.prod([len(c) for c in per_pos], dtype=np.float64))
    if method == "auto":
        method = "enumerate" if count <= ENUMERATE_LIMIT else "best_first"
    if method == "enumerate":
        combos = [(tup, score(tup)) for tup in itertools.product(*per_pos)]
        combos.sort(key=lambda c: (-c[1], c[0]))
        return combos[:budget]
    if count == 0:
        return []
    avail = [len(c) for c in per_pos]  # finite slots come first in each row
    start = (0,) * D
    heap = [(-score(start), start, 0)]
    out = []
    while heap and len(out) < budget:
        neg, tup, last = heapq.heappop(heap)
        out.append((tup, -neg))
        for j in range(last, D):
            if tup[j] + 1 < avail[j]:
                nxt = tup[:j] + (tup[j] + 1,) + tup[j + 1:]
                heapq.heappush(heap, (-score(nxt), nxt, j))
    return out


def tree_max_nodes(depth: int, budget: int) -> int:
    """Upper bound on the node count of a tree: the root plus one node per
    position of every kept sequence."""
    return 1 + depth * budget


def tree_build(ids, logq, budget: int):
    """The candidate tree of every sequence (readings T3, T4).

    ids, logq [B, D, top_k] from ``tree_topk``. Returns a dict of
      node_token  [B, N] int32  token of the node (root and padding: -1)
      node_parent [B, N] int32  parent node (root and padding: -1)
      node_depth  [B, N] int32  0 for the root, j for a prefix of length j
                                (padding: -1)
      n_nodes     [B]    int32
      kept        list per sequence of (rank tuple, joint log-probability)
    with N = tree_max_nodes(D, budget).
    """
    ids = np.asarray(ids)
    B, D, _ = ids.shape
    N = tree_max_nodes(D, budget)
    node_token = np.full((B, N), -1, dtype=np.int32)
    node_parent = np.full((B, N), -1, dtype=np.int32)
    node_depth = np.full((B, N), -1, dtype=np.int32)
    n_nodes = np.zeros(B, dtype=np.int32)
    kept_all = []
    for b in range(B):
        kept = tree_candidates(logq[b], budget)
        kept_all.append(kept)
        prefixes = sorted({tup[:j] for tup, _ in kept for j in range(1, D + 1)},
                          key=lambda t: (len(t), t))
        index = {(): 0}
        node_depth[b, 0] = 0
        for n, pre in enumerate(prefixes, start=1):
            index[pre] = n
            node_parent[b, n] = index[pre[:-1]]
            node_depth[b, n] = len(pre)
            node_token[b, n] = ids[b, len(pre) - 1, pre[-1]]
        n_nodes[b] = 1 + len(prefixes)
    return {"node_token": node_token, "node_parent": node_parent,
            "node_depth": node_depth, "n_nodes": n_nodes, "kept": kept_all}


def tree_draft(q_logits, top_k: int, budget: int):
    """Top-k candidates, then the tree: ``tree_build(*tree_topk(q), budget)``."""
    ids, logq = tree_topk(q_logits, top_k)
    tree = tree_build(ids, logq, budget)
    tree["topk_ids"], tree["topk_logq"] = ids, logq
    return tree


def tree_verify_u(p_logits, node_token, node_parent, n_nodes, u):
    """Walk each sequence's tree with the AR rows (readings T5, T6).

    p_logits [B, N, V]: row n = the AR logits after node n's prefix (rows at
    or beyond n_nodes[b] are not read). u [B, D+1]: the sampling uniform of
    each depth, D = the tree depth (u.shape[1] - 1).

    Returns a dict of out_tokens [B, D+1] int32 (-1 padded), accepted_len
    [B] int32 (accepted tree tokens, 0..D, or -1), and per depth the draw
    boundaries (c_prev, c_at, threshold, total, each [B, D+1], NaN where no
    draw happened) for near-tie accounting.
    """
    p = np.asarray(p_logits, dtype=np.float64)
    B, N, V = p.shape
    u = np.asarray(u, dtype=np.float64)
    D = u.shape[1] - 1
    out = np.full((B, D + 1), -1, dtype=np.int32)
    acc = np.zeros(B, dtype=np.int32)
    bounds = {k: np.full((B, D + 1), np.nan) for k in ("c_prev", "c_at", "threshold", "total")}
    for b in range(B):
        node = 0
        for j in range(D + 1):
            row = p[b, node]
            fin = np.isfinite(row)
            if not fin.any():
                out[b, :] = -1
                acc[b] = -1
                break
            w = np.where(fin, np.exp(row - row[fin].max()), 0.0)
            idx, c_prev, c_at, t, total = _inverse_cdf(w[None, :], u[b, j:j + 1])
            y = int(idx[0])
            for key, val in (("c_prev", c_prev), ("c_at", c_at), ("threshold", t),
                             ("total", total)):
                bounds[key][b, j] = val[0]
            out[b, j] = y
            child = [c for c in range(1, int(n_nodes[b]))
                     if node_parent[b, c] == node and node_token[b, c] == y]
            if not child:
                acc[b] = j
                break
            node = child[0]
        else:  # pragma: no cover  (a leaf has no children, so the loop breaks)
            acc[b] = D
    res = {"out_tokens": out, "accepted_len": acc}
    res.update(bounds)
    return res


def tree_uniforms(B: int, D: int, seed: int, step: int):
    """Sampling uniforms of depths 0..D: word 1 of the Philox block of
    (b, j, step), as the linear verifier's sampling uniforms."""
    return uniforms_for_block(B, D, seed, step)[1]


def tree_verify(p_logits, tree, seed: int, step: int):
    """``tree_verify_u`` with ``tree_uniforms``, for a tree from
    ``tree_draft`` (its ``topk_ids`` give the depth D)."""
    D = np.asarray(tree["topk_ids"]).shape[1]
    B = np.asarray(tree["node_token"]).shape[0]
    return tree_verify_u(p_logits, tree["node_token"], tree["node_parent"], tree["n_nodes"],
                         tree_uniforms(B, D, seed, step))
