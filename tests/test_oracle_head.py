"""Pins of the oracle for the LM head fused with the verifier's statistics.

The fused row adds no arithmetic of its own to the method: the verifier's row
normalisers are computed where the LM head writes the logits, as per-tile
partials, and the verifier reads p and q in the LM head's row layout. So the
pins check (i) the partials against library logsumexp and closed forms, and
(ii) the layout reading against hand-built p and q.
"""
import numpy as np
import pytest
from scipy import special

from oracle import merge_row_stats, row_stat_partials, verify_block, verify_block_head

LOG2E = 1.0 / np.log(2.0)


@pytest.mark.parametrize("N,tile", [(1000, 256), (256, 256), (37, 7), (5, 1), (300, 300)])
def test_merged_partials_are_logsumexp(N, tile):
    rng = np.random.default_rng(N + tile)
    y = rng.normal(0, 3, size=(6, N))
    y[1, : N // 2] = -np.inf          # masked entries
    y[2, :] = -40.0                   # a flat row
    st = row_stat_partials(y, tile)
    assert st.shape == (6, (N + tile - 1) // tile, 2)
    got = merge_row_stats(st)
    want = special.logsumexp(y, axis=1)
    assert np.allclose(got, want, rtol=0, atol=1e-12 * max(1.0, np.abs(want).max()))


def test_partials_closed_forms():
    y = np.array([[1.0, 2.0, 3.0, -np.inf, 0.5]])
    st = row_stat_partials(y, 2)
    # tile maxima times log2(e); an all-masked tile is (-inf, 0)
    assert np.allclose(st[0, :, 0], [2.0 * LOG2E, 3.0 * LOG2E, 0.5 * LOG2E])
    # a tile of one finite value has z = 1; (1, 2) has z = 2^-log2e + 1 = 1/e + 1
    assert st[0, 1, 1] == 1.0 and st[0, 2, 1] == 1.0
    assert np.isclose(st[0, 0, 1], 1.0 + np.exp(-1.0))
    masked = row_stat_partials(np.full((1, 4), -np.inf), 2)
    assert np.all(np.isneginf(masked[..., 0])) and np.all(masked[..., 1] == 0.0)
    assert np.isneginf(merge_row_stats(masked)[0])


def test_partials_are_shift_equivariant():
    rng = np.random.default_rng(3)
    y = rng.normal(size=(3, 600))
    a = merge_row_stats(row_stat_partials(y))
    b = merge_row_stats(row_stat_partials(y + 7.25))
    assert np.allclose(b - a, 7.25, atol=1e-12)


def _blocks(B, K, V, seed):
    rng = np.random.default_rng(seed)
    y_ar = rng.normal(0, 2, size=(B * (K + 1), V))
    y_dr = y_ar + rng.normal(0, 0.7, size=y_ar.shape)
    x = rng.integers(0, V, size=(B, K)).astype(np.int32)
    return y_ar, y_dr, x


def test_head_layout_matches_hand_built_p_and_q():
    B, K, V = 3, 4, 50
    y_ar, y_dr, x = _blocks(B, K, V, 5)
    p = np.zeros((B, K + 1, V))
    q = np.zeros((B, K, V))
    for b in range(B):
        for i in range(K + 1):
            p[b, i] = y_ar[b * (K + 1) + i]
        for i in range(K):
            q[b, i] = y_dr[b * (K + 1) + i]
    got = verify_block_head(y_ar, y_dr, x, seed=9, step=2)
    want = verify_block(p, q, x, seed=9, step=2)
    for key in ("out_tokens", "accepted_len"):
        assert np.array_equal(got[key], want[key])


def test_head_layout_ignores_the_bonus_rows_draft_output():
    B, K, V = 4, 3, 40
    y_ar, y_dr, x = _blocks(B, K, V, 6)
    a = verify_block_head(y_ar, y_dr, x, seed=1, step=0)
    y2 = y_dr.copy()
    y2[K::K + 1] = 1e3  # row K of every block: never a draft distribution
    b = verify_block_head(y_ar, y2, x, seed=1, step=0)
    assert np.array_equal(a["out_tokens"], b["out_tokens"])
    # while the AR row of the same position is the bonus distribution
    y3 = y_ar.copy()
    y3[K::K + 1] = -1e3
    y3[K::K + 1, 7] = 1e3  # bonus token 7 with certainty
    c = verify_block_head(y3, y_dr, x, seed=1, step=0)
    full = c["accepted_len"] == K
    assert np.all(c["out_tokens"][full, K] == 7)
