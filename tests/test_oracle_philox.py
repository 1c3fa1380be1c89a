"""Pins of the oracle's Philox4x32-10 and uniform mapping.

Philox4x32-10 is the counter-based generator of Salmon et al., "Parallel
Random Numbers: As Easy as 1, 2, 3" (SC'11). The oracle's stream is pinned to
the known-answer vectors published with that paper's Random123 library
(tests/golden/philox_kat.json), so a wrong multiplier, Weyl constant, word
order or round count fails here. The other tests pin the structure (10
invertible rounds with the stated key schedule, checked by running the rounds
backwards) and the statistical quality the sampler's losslessness needs
(uniform, independent words and counters).
"""

import json
import os

import numpy as np
import pytest
from scipy import stats

from oracle import philox4x32_10, uniforms_for_block, word_to_uniform

MASK = (1 << 32) - 1
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox_kat.json")


def _kat_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _kat_cases(), ids=lambda c: c["name"])
def test_published_known_answer_vectors(case):
    ctr = np.array([int(w, 16) for w in case["counter"]], dtype=np.uint32)
    key = np.array([int(w, 16) for w in case["key"]], dtype=np.uint32)
    out = philox4x32_10(ctr, key)
    assert [f"{int(w):08x}" for w in out] == case["out"]
    # batched calls see the same block
    both = philox4x32_10(np.stack([ctr, ctr]), key)
    assert np.array_equal(both[0], out) and np.array_equal(both[1], out)


def test_block_words_map_to_the_documented_counter_and_key():
    # counter (b, i, step lo, step hi), key (seed lo, seed hi): the all-zero
    # known answer is sequence 0, position 0, step 0 under seed 0
    zeros = next(c for c in _kat_cases() if c["name"] == "zeros")
    u_acc, u_smp = uniforms_for_block(B=1, K=1, seed=0, step=0)
    assert u_acc[0, 0] == (int(zeros["out"][0], 16) >> 8) * 2.0**-24
    assert u_smp[0, 0] == (int(zeros["out"][1], 16) >> 8) * 2.0**-24
    pi = next(c for c in _kat_cases() if c["name"] == "pi digits")
    seed = int(pi["key"][0], 16) | (int(pi["key"][1], 16) << 32)
    step = int(pi["counter"][2], 16) | (int(pi["counter"][3], 16) << 32)
    ctr = np.array([[int(pi["counter"][0], 16), int(pi["counter"][1], 16),
                     step & MASK, step >> 32]], dtype=np.uint32)
    key = np.array([seed & MASK, seed >> 32], dtype=np.uint32)
    assert [f"{int(w):08x}" for w in philox4x32_10(ctr, key)[0]] == pi["out"]


def _inv_mod32(a: int) -> int:
    return pow(a, -1, 1 << 32)


def _philox_backwards(out, key, M0, M1, W0, W1, rounds=10):
    """Undo ``rounds`` Philox rounds in plain Python integers.

    A forward round sends (c0, c1, c2, c3) to
    (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)).
    Since M0 and M1 are odd, lo(M c) determines c; the xors then give back
    c1 and c3.
    """
    o0, o1, o2, o3 = (int(v) for v in out)
    k0, k1 = int(key[0]), int(key[1])
    iM0, iM1 = _inv_mod32(M0), _inv_mod32(M1)
    for r in reversed(range(rounds)):
        rk0 = (k0 + r * W0) & MASK
        rk1 = (k1 + r * W1) & MASK
        c2 = (o1 * iM1) & MASK
        c0 = (o3 * iM0) & MASK
        hi1 = (M1 * c2) >> 32
        hi0 = (M0 * c0) >> 32
        c1 = o0 ^ hi1 ^ rk0
        c3 = o2 ^ hi0 ^ rk1
        o0, o1, o2, o3 = c0, c1, c2, c3
    return (o0, o1, o2, o3)


def test_rounds_invert_to_the_counter():
    # Multipliers and Weyl constants of Philox4x32 as given in SC'11.
    M0, M1, W0, W1 = 0xD2511F53, 0xCD9E8D57, 0x9E3779B9, 0xBB67AE85
    rng = np.random.default_rng(5)
    ctr = rng.integers(0, 1 << 32, size=(64, 4), dtype=np.uint64).astype(np.uint32)
    key = rng.integers(0, 1 << 32, size=(64, 2), dtype=np.uint64).astype(np.uint32)
    out = philox4x32_10(ctr, key)
    for j in range(64):
        back = _philox_backwards(out[j], key[j], M0, M1, W0, W1)
        assert back == tuple(int(v) for v in ctr[j])


def test_deterministic_and_broadcast():
    ctr = np.array([[1, 2, 3, 4], [5, 6, 7, 8]], dtype=np.uint32)
    key = np.array([9, 10], dtype=np.uint32)
    a = philox4x32_10(ctr, key)
    b = np.stack([philox4x32_10(ctr[i], key) for i in range(2)])
    assert np.array_equal(a, b)
    assert np.array_equal(a, philox4x32_10(ctr, key))
    # A different key gives a different block.
    assert not np.array_equal(a, philox4x32_10(ctr, key + 1))


def test_uniform_grid_and_range():
    w = np.array([0, 255, 256, 0xFFFFFFFF, 0x80000000], dtype=np.uint32)
    u = word_to_uniform(w)
    assert u[0] == 0.0 and u[1] == 0.0
    assert u[2] == 2.0**-24
    assert u[3] == 1.0 - 2.0**-24
    assert u[4] == 0.5
    # Every value is exactly a float32 too.
    assert np.array_equal(u.astype(np.float32).astype(np.float64), u)


def test_uniforms_are_uniform_and_independent():
    u_acc, u_smp = uniforms_for_block(B=1 << 14, K=63, seed=12345, step=7)
    a = u_acc.ravel()
    s = u_smp[:, :63].ravel()
    for v in (a, s):
        counts, _ = np.histogram(v, bins=256, range=(0.0, 1.0))
        assert stats.chisquare(counts).pvalue > 1e-3
        assert abs(v.mean() - 0.5) < 5 * np.sqrt(1 / 12 / v.size)
    # The two words of a block are uncorrelated; so are neighbouring counters.
    n = a.size
    assert abs(np.corrcoef(a, s)[0, 1]) < 5 / np.sqrt(n)
    assert abs(np.corrcoef(a[:-1], a[1:])[0, 1]) < 5 / np.sqrt(n)
    # Neighbouring steps and seeds give unrelated streams.
    a2, _ = uniforms_for_block(B=1 << 14, K=63, seed=12345, step=8)
    a3, _ = uniforms_for_block(B=1 << 14, K=63, seed=12346, step=7)
    assert abs(np.corrcoef(a, a2.ravel())[0, 1]) < 5 / np.sqrt(n)
    assert abs(np.corrcoef(a, a3.ravel())[0, 1]) < 5 / np.sqrt(n)


def test_avalanche():
    rng = np.random.default_rng(1)
    ctr = rng.integers(0, 1 << 32, size=(4096, 4), dtype=np.uint64).astype(np.uint32)
    key = np.array([77, 88], dtype=np.uint32)
    out = philox4x32_10(ctr, key)
    flips = []
    for word in range(4):
        for bit in (0, 13, 31):
            c2 = ctr.copy()
            c2[:, word] ^= np.uint32(1 << bit)
            d = philox4x32_10(c2, key) ^ out
            flips.append(np.unpackbits(d.view(np.uint8), axis=None).sum() / d.shape[0])
    flips = np.array(flips)
    assert np.all(np.abs(flips - 64.0) < 1.0)


@pytest.mark.parametrize("step", [0, 1, (1 << 32) + 3])
def test_step_high_bits_matter(step):
    a, _ = uniforms_for_block(4, 4, seed=3, step=step)
    b, _ = uniforms_for_block(4, 4, seed=3, step=step ^ (1 << 40))
    assert not np.array_equal(a, b)
