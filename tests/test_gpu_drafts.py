"""Parity of the CUDA draft sampler (linear Psi-Spec proposal) with the
float64 oracle, on a B200.

Drafted ids must equal the oracle's, except draws whose threshold lies
within the verifier's near-tie band of a CDF boundary (counted). Covers V = 1,
odd V (unaligned rows), -inf masks, a row with no finite logit, bf16 and f32,
the Qwen3-8B vocabulary at B = 64, K = 16, and a chi-square test of device
draws against softmax(q).
"""
import numpy as np
import pytest
import torch
from scipy.special import softmax as sp_softmax
from scipy.stats import chisquare

import oracle
from lossless_decoding_b200.inputs import verify_inputs
from tests.parity import compare_drafts, widen

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_decoding_b200 import api as A
    return A


def _check(api, q, seed, step, rows=None):
    got = api.sample_drafts(q, seed, step)
    torch.cuda.synchronize()
    B, K, _ = q.shape
    u = oracle.draft_uniforms(B, K, seed, step)
    sel = np.arange(B) if rows is None else np.asarray(rows)
    ids, det = oracle.sample_drafts_u(widen(q[torch.as_tensor(sel, device=q.device)]), u[sel])
    return compare_drafts(got.cpu().numpy()[sel], ids, det)


@pytest.mark.parametrize("B,K,V,dtype,dist", [
    (1, 8, 4096, "f32", "normal"),
    (3, 2, 1, "bf16", "normal"),       # V = 1
    (4, 3, 7, "f32", "normal"),        # V below one vector
    (5, 4, 4097, "bf16", "gumbel"),    # odd V: rows not 16-byte aligned
    (16, 16, 32000, "bf16", "gumbel"),
    (64, 4, 1000, "f32", "normal"),
])
def test_parity_small(api, B, K, V, dtype, dist):
    for seed, step in ((0, 0), (99, 12)):
        v = verify_inputs(B, K, V, dtype=dtype, dist=dist, seed=seed + V, device=DEV)
        compared, ties = _check(api, v.q_logits, seed, step)
        assert compared + ties == B * K


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_parity_qwen3_vocabulary_batched(api, dtype):
    """B = 64, K = 16 over V = 151936; the oracle checks 8 sequences (128
    draws). The draft band (TAU_DRAFT of the total, derived from the sampler's
    arithmetic) leaves only draws very close to a CDF boundary uncompared: at
    least 90% of the draws are compared token for token, and all of them must
    match."""
    v = verify_inputs(64, 16, 151936, dtype=dtype, dist="normal", seed=3, device=DEV)
    compared, ties = _check(api, v.q_logits, 1234, 5, rows=[0, 1, 9, 17, 31, 40, 55, 63])
    print(f"draft parity {dtype}: {compared} compared, {ties} near ties of {8 * 16}")
    assert compared + ties == 8 * 16
    assert compared >= int(np.ceil(0.9 * 8 * 16))


@pytest.mark.parametrize("dist,sigma", [("gumbel", 0.25), ("gumbel", 4.0)])
def test_parity_full_vocabulary_gumbel(api, dist, sigma):
    """The sweep's boosted-Gumbel rows at V = 151936 (bf16): at least 90% of
    the 4 x 16 draws compared, all equal."""
    v = verify_inputs(4, 16, 151936, dtype="bf16", dist=dist, sigma=sigma, seed=9, device=DEV)
    compared, ties = _check(api, v.q_logits, 77, 2, rows=[0, 1, 2, 3])
    print(f"draft parity gumbel sigma={sigma}: {compared} compared, {ties} near ties of 64")
    assert compared + ties == 4 * 16
    assert compared >= int(np.ceil(0.9 * 4 * 16))


def test_masks_and_empty_rows(api):
    g = torch.Generator().manual_seed(4)
    q = torch.randn(6, 5, 300, generator=g)
    q[..., :150] = float("-inf")
    q[2, 3, :] = float("-inf")  # no distribution at all
    qd = q.to(DEV)
    got = api.sample_drafts(qd, 8, 1)
    torch.cuda.synchronize()
    got = got.cpu()
    assert got[2, 3] == -1
    mask = torch.ones_like(got, dtype=torch.bool)
    mask[2, 3] = False
    assert torch.all(got[mask] >= 150)
    compare_drafts(got.numpy(), *oracle.sample_drafts(q.double().numpy(), 8, 1))


def test_chisquare_on_device(api):
    V, B, K = 10, 1 << 15, 32
    rng = np.random.default_rng(6)
    row = rng.standard_normal(V).astype(np.float32) * 1.3
    q = torch.from_numpy(np.broadcast_to(row, (B, K, V)).copy()).to(DEV)
    got = api.sample_drafts(q, 2024, 77)
    torch.cuda.synchronize()
    counts = np.bincount(got.cpu().numpy().reshape(-1), minlength=V)
    expected = sp_softmax(row.astype(np.float64)) * B * K
    assert chisquare(counts, expected).pvalue > 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_blocks_of_k_plus_one_rows_read_in_place(api, dtype):
    """Drawing the first K rows of each block of K + 1 (the LM head's
    draft-pathway layout) gives the ids of the same rows copied out
    contiguously, bit for bit: same rows, same counters."""
    B, K, V = 6, 5, 3001
    v = verify_inputs(B, K + 1, V, dtype=dtype, dist="gumbel", sigma=1.0, seed=31, device=DEV)
    blocks = v.p_logits  # [B, K + 2, V]: any block of at least K + 1 rows works
    R = blocks.shape[1]
    got = api.sample_drafts(blocks, 77, 3, num_drafts=K)
    ref = api.sample_drafts(blocks[:, :K].contiguous(), 77, 3)
    torch.cuda.synchronize()
    assert got.shape == (B, K) and R > K
    assert torch.equal(got, ref)
