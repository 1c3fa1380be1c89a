"""The draft sampler's near-tie band covers the sampler's own roundings.

tests/parity.py excludes a drafted id from the comparison when the oracle's
threshold u * total lies within TAU_DRAFT * spread of a CDF boundary, spread
= sqrt(sum_i w_i^2) of the row's weights. This test
replays, in numpy float32, the roundings the device's sampler makes on rows
shaped like the full-vocabulary test workloads, with the SFU's 2^(.) error
injected at its measured largest relative size (1.46e-7):

  * pass 1, per chunk (2048 bfloat16 or 1024 float32 logits) and per lane:
    the reference m kept at the running maximum (each group of two vectors
    moves it up to its own maximum first, rescaling the sum by an SFU
    2^(m - gm)), the exponent argument x log2 e - m by one fused multiply-add,
    2^(.) on the SFU, the group's weights summed as a tree of float32 pairs,
    the lane's sum accumulated in float32 group by group; then the warp's
    pair: the lanes' sums rescaled to the warp's maximum and added in
    float64;
  * pass 2: each chunk's sum rescaled to the largest maximum M in float64
    and accumulated in float64;
  * pass 3: the chosen chunk's weights 2^(x log2 e - M) token by token in
    float64 (the SFU again);

and checks that the comparison of the running sum with u * total moves by at
most a third of the band, for every drawn token of six workloads from
diffuse to concentrated rows.
"""

import numpy as np
import pytest

import oracle
from lossless_decoding_b200.inputs import verify_inputs
from tests.parity import TAU_DRAFT, widen

F32 = np.float32
LOG2E = F32(1.4426950408889634)
SFU_REL = 1.46e-7
LANES, ROUNDS, KV = 32, 2, 4   # a chunk: ROUNDS rounds of KV 16-byte vectors per lane


def _sfu(a, rng):
    """2^a in float32 with the SFU's error (exact where a is 0)."""
    a64 = a.astype(np.float64)
    y = np.exp2(a64) * (1.0 + np.where(a64 == 0.0, 0.0, rng.uniform(-SFU_REL, SFU_REL, a.shape)))
    return y.astype(F32)


def _arg(x, m):
    """fmaf(x, log2 e, -m): exact product and sum in float64, one rounding."""
    return (x.astype(np.float64) * np.float64(LOG2E) - np.asarray(m, np.float64)).astype(F32)


def _tree(w):
    """The weights of one fold [..., n] (pair i = elements 2i, 2i+1) summed
    as the packed tree: pairs added halfwise level by level, then lo + hi."""
    p = w.reshape(w.shape[:-1] + (w.shape[-1] // 2, 2))
    while p.shape[-2] > 1:
        p = (p[..., 0::2, :] + p[..., 1::2, :]).astype(F32)
    return (p[..., 0, 0] + p[..., 0, 1]).astype(F32)


def _device_draw_boundaries(row, u, y, kvec, rng):
    """Device-side running sums just before and after token y, and u * total
    (kvec logits per 16-byte vector: 8 for bfloat16, 4 for float32)."""
    V = row.size
    L = ROUNDS * KV * LANES * kvec  # logits per chunk
    n_chunks = (V + L - 1) // L
    pad = n_chunks * L - V
    x = np.concatenate([row, np.full(pad, -np.inf, F32)]).reshape(n_chunks, ROUNDS, KV, LANES, kvec)
    # per lane, folds of two vectors in round order
    x = x.transpose(0, 3, 1, 2, 4).reshape(n_chunks, LANES, ROUNDS * 2, 2 * kvec)
    # the lane's reference is its running maximum: each group moves it up to
    # the group's maximum (rescaling the sum by an SFU 2^(m - gm)) before its
    # weights are summed
    m = np.full((n_chunks, LANES), -np.inf, F32)
    z = np.zeros((n_chunks, LANES), F32)
    for g in range(ROUNDS * 2):
        grp = x[:, :, g, :]
        gm = (np.max(grp, axis=-1) * LOG2E).astype(F32)
        up = np.isfinite(gm) & (gm > m)
        resc = np.where(np.isfinite(m), (z * _sfu(np.where(np.isfinite(m) & up, m - gm, 0), rng)).astype(F32), F32(0))
        z = np.where(up, resc, z).astype(F32)
        m = np.where(up, gm, m).astype(F32)
        a = _arg(grp, np.where(np.isfinite(m), m, 0)[..., None])
        ok = np.isfinite(a) & np.isfinite(m)[..., None]
        w = np.where(ok, _sfu(np.where(ok, a, 0), rng), F32(0))
        z = (z + _tree(w)).astype(F32)
    # the warp's pair: lane sums rescaled to the warp's maximum in float64
    mm = m.max(axis=1)
    lane_w = np.where(np.isfinite(m), z.astype(np.float64) * np.exp2(m.astype(np.float64) - mm[:, None].astype(np.float64)), 0.0)
    cs, cm = lane_w.sum(axis=1), mm
    M = cm.max()
    wc = cs * np.exp2(cm.astype(np.float64) - np.float64(M))  # float64 rescale
    total = wc.sum()
    c0 = (y // L) * L
    wt = _sfu(_arg(row[c0:y + 1], M), rng).astype(np.float64)
    before = wc[: y // L].sum() + wt[:-1].sum()
    return before, before + wt[-1], float(u) * total, total


@pytest.mark.parametrize("dist,sigma,dtype,seed", [
    ("normal", 1.0, "bf16", 3), ("gumbel", 0.25, "bf16", 4), ("gumbel", 4.0, "f32", 5),
    ("normal", 0.5, "bf16", 7), ("gumbel", 1.0, "bf16", 8), ("normal", 2.0, "f32", 9)])
def test_band_covers_the_sampler_roundings(dist, sigma, dtype, seed):
    B, K, V = 4, 8, 151936
    rng = np.random.default_rng(seed)
    v = verify_inputs(B, K, V, dtype=dtype, dist=dist, sigma=sigma, seed=seed)
    q = widen(v.q_logits)
    u = oracle.draft_uniforms(B, K, 1234, 5)
    ids, det = oracle.sample_drafts_u(q, u)
    worst = 0.0
    for b in range(B):
        for i in range(K):
            row = q[b, i].astype(F32)
            y = int(ids[b, i])
            before, at, t, tot = _device_draw_boundaries(row, u[b, i], y,
                                                         8 if dtype == "bf16" else 4, rng)
            scale = tot / det["total"][b, i]
            t_o = det["threshold"][b, i]
            d_prev = (before - t) / scale - (det["c_prev"][b, i] - t_o)
            d_at = (at - t) / scale - (det["c_at"][b, i] - t_o)
            worst = max(worst, max(abs(d_prev), abs(d_at)) / det["spread"][b, i])
    print(f"{dist} sigma={sigma} {dtype}: largest move {worst:.2e} of the spread")
    assert worst < TAU_DRAFT / 3, f"the sampler's roundings moved the comparison by {worst:.2e}"
