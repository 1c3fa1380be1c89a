"""The verifier's near-tie band for draws covers the draw's own roundings.

tests/parity.py excludes a verifier draw from the token comparison when the
oracle's threshold u' * total lies within TAU_DRAW * (total + q_res) of a CDF
boundary. This test replays, in numpy float32, the roundings the device's
draw makes -- the exponent argument from three FMA roundings, the SFU's
2^(.) with its measured largest relative error (1.46e-7) injected as noise,
a float32 tree over each 16-byte vector of eight weights, float64 beyond,
and row normalisers perturbed at the float32 level -- on rows shaped like
the full-vocabulary test workloads, and checks that the comparison of the
running sum with u' * total moves by at most a third of the band.
"""

import numpy as np
import pytest

import oracle
from lossless_decoding_b200.inputs import verify_inputs
from tests.parity import TAU_DRAW, widen

F32 = np.float32
LOG2E = 1.4426950408889634074
CHI = F32(LOG2E)
CLO = F32(LOG2E - float(CHI))
SFU_REL = 1.46e-7


def _fmaf(x, y, z):
    """float32 fused multiply-add: exact product and sum in float64, one rounding."""
    return (x.astype(np.float64) * np.float64(y) + z.astype(np.float64)).astype(F32)


def _device_weights(logits: np.ndarray, L: float, rng) -> tuple:
    """Exponent arguments and weights 2^(l log2 e - L) as the device forms them."""
    hi = F32(L)
    lo = F32(L - float(hi))
    a = (_fmaf(logits, CLO, _fmaf(logits, CHI, np.full_like(logits, -hi))) - lo).astype(F32)
    w = np.exp2(a.astype(np.float64)) * (1.0 + rng.uniform(-SFU_REL, SFU_REL, a.shape))
    return a, w.astype(F32)


def _vector_sums(w: np.ndarray) -> np.ndarray:
    """Sums of eight consecutive weights as a float32 tree, as float64."""
    n = (w.size + 7) // 8 * 8
    v = np.zeros(n, F32)
    v[: w.size] = w
    v = v.reshape(-1, 8)
    v = (v[:, 0::2] + v[:, 1::2]).astype(F32)
    v = (v[:, 0::2] + v[:, 1::2]).astype(F32)
    return (v[:, 0] + v[:, 1]).astype(np.float64)


@pytest.mark.parametrize("dist,sigma,dtype,seed", [
    ("normal", 1.0, "bf16", 1), ("gumbel", 0.25, "bf16", 2), ("gumbel", 4.0, "f32", 3)])
def test_band_covers_the_draw_roundings(dist, sigma, dtype, seed):
    B, K, V = 6, 8, 151936
    rng = np.random.default_rng(seed)
    v = verify_inputs(B, K, V, dtype=dtype, dist=dist, sigma=sigma, seed=seed)
    p_log, q_log = widen(v.p_logits), widen(v.q_logits)
    ref = oracle.verify_block(p_log, q_log, v.draft_tokens.numpy(), seed=seed, step=0)
    worst = 0.0
    for b in range(B):
        n = int(ref["accepted_len"][b])
        lp = p_log[b, n].astype(F32)
        Lp = np.log2(np.sum(np.exp2(lp.astype(np.float64) * LOG2E))) + rng.normal(0, 1e-7)
        ap, wp = _device_weights(lp, Lp, rng)
        if n < K:
            lq = q_log[b, n].astype(F32)
            Lq = np.log2(np.sum(np.exp2(lq.astype(np.float64) * LOG2E))) + rng.normal(0, 1e-7)
            aq, wq = _device_weights(lq, Lq, rng)
            w = np.where(ap > aq, np.maximum(F32(0), (wp - wq).astype(F32)), F32(0))
        else:
            w = wp
        # running sums at the boundaries of the oracle's token: chunk sums of
        # vector sums before its chunk, then token by token, in float64
        y = int(ref["out_tokens"][b, n])
        vec = _vector_sums(w)
        tot_dev = vec.sum()
        c0 = (y // 256) * 256  # the device's chunk of 256 tokens holding y: summed token by token
        before = vec[: c0 // 8].sum() + w[c0:y].astype(np.float64).sum()
        at = before + float(w[y])
        tot, t = ref["cdf_total"][b], ref["cdf_t"][b]
        u = t / tot
        scale = tot_dev / tot
        d_prev = (before - u * tot_dev) / scale - (ref["cdf_prev"][b] - t)
        d_at = (at - u * tot_dev) / scale - (ref["cdf_at"][b] - t)
        worst = max(worst, max(abs(d_prev), abs(d_at)) / (tot + ref["cdf_qres"][b]))
    assert worst < TAU_DRAW / 3, f"draw roundings moved the comparison by {worst:.2e}"
