"""Plain, slow, float64 CPU oracle for one Psi-Spec decode step.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import, call or run this module. The
CUDA library (``lossless_decoding_b200``) never imports it and this module
imports nothing from that package; the two share no code, tables or
constants. Its arithmetic is float64 throughout.

Sources (the pages on "Unlocking Lossless Speedups in LLMs via Discrete
Diffusion", Uno):

* [SUM]    the picx.dev summary page of the paper, sections "Methodology /
           Architecture: Diffusion-Augmented LLMs" and "Methodology /
           Psi-Speculative Sampler".
* [READER] the paperglide reader page "Unlocking Lossless Speedups in LLMs
           via Discrete Diffusion", sections "The Uno Framework", "The
           Psi-Speculative Sampler" and "Sampler Extensions" (linear sampler).
* [SC11]   Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
           1, 2, 3", SC'11 -- the Philox4x32-10 counter-based generator.
* [SD]     the standard speculative-sampling rule the pages cite (Leviathan et
           al. 2023; Chen et al. 2023): accept drafted token x_i while
           u_i < p_i(x_i) / q_i(x_i); at the first rejection draw one token
           from norm(max(0, p - q)); if every draft is accepted draw one more
           token from the verifier's next distribution.

What each function follows:

* ``dualpath_linear``: [SUM] Architecture and [READER] "The Uno Framework":
  frozen AR weights are shared; drafting adds a LoRA adapter (rank r, scale
  alpha/r; rank 128, alpha 256 on the pages), verification uses the AR
  weights alone. y_AR = x W^T and y_draft = y_AR + T B^T with
  T = (alpha/r) x A^T.
* ``verify_block`` / ``verify_block_u``: [READER] "The Psi-Speculative
  Sampler" (verify each prefix with the frozen AR model, keep the longest
  accepted prefix, and if all drafts are accepted emit one more token from
  the AR verifier) and "Sampler Extensions" (the linear sampler either
  accepts the whole block or replaces the tail with a single token drawn
  from the verifier), with the accept and residual rules of [SD].
* ``philox4x32_10``: [SC11].
* ``row_stat_partials`` / ``merge_row_stats`` / ``verify_block_head``: the
  verifier's row normalisers split into per-column-tile partials (the form in
  which the LM head can produce them) and the verifier on the LM head's row
  layout (p = a block's K+1 AR rows, q_i = its draft row i < K); no new
  arithmetic, the definitions above rearranged.

Readings of the pages that this module fixes (each one is listed with its
reason in the repository's design notes):

1. Accept test: ``u * q_i(x_i) < p_i(x_i)``, strict. Identical to
   u < p/q for q > 0; for q = 0 it accepts iff p > 0.
2. Uniforms: Philox4x32-10 with key (seed lo, seed hi) and counter
   (b, i, step lo, step hi). Output word 0 is the accept uniform of
   position i; word 1 is the sampling uniform used when position i is
   where the residual (or, for i = K, the bonus) token is drawn.
   u = (word >> 8) * 2^-24, exactly representable in float32 and float64.
3. p carries K+1 rows per sequence: row K is the verifier's distribution
   after the last draft, used for the bonus token.
4. Inverse CDF: y = the smallest v with C_v > u' * C_{V-1}, where C is the
   running sum of the (unnormalised) sampling weights in index order. If
   rounding leaves no such v, y = the largest v with positive weight.
5. If the residual mass sum_v max(0, p - q) is zero at a rejected position
   (possible only through rounding), sample from p at that position.
6. Temperature is 1 (all evaluations on the pages use temperature 1).
7. A draft id outside [0, V) anywhere in a sequence's block marks that
   sequence invalid: accepted length -1 and all output tokens -1.
8. The adapter input T is rounded to bfloat16 (round to nearest, ties to
   even) when the operands are bfloat16, because the adapter product is a
   bfloat16 tensor-core product; with float32 operands T is not rounded.
"""

from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# bfloat16 (exact widening and round-to-nearest-even), from the IEEE-754
# binary32 layout: bfloat16 is the top 16 bits of a binary32.
# --------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bfloat16 bit patterns (uint16) to float64 exactly."""
    b = np.asarray(bits).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps 8 significant bits. With x = f * 2^e and f in [0.5, 1)
    (``np.frexp``, exact), the spacing of representable values near x is
    2^(e-8); ``np.rint`` rounds half to even. Finite inputs of normal
    magnitude only (the oracle never produces others).
    """
    x = np.asarray(x, dtype=np.float64)
    f, e = np.frexp(x)
    scaled = np.ldexp(f, 8)  # in [128, 256) in magnitude, exact
    return np.ldexp(np.rint(scaled), e - 8)


# --------------------------------------------------------------------------
# Philox4x32-10 [SC11]
# --------------------------------------------------------------------------

_MASK32 = np.uint64(0xFFFFFFFF)
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint64(0x9E3779B9)
_PHILOX_W1 = np.uint64(0xBB67AE85)

PHILOX_WORD_ACCEPT = 0
PHILOX_WORD_SAMPLE = 1
PHILOX_WORD_DRAFT = 2  # drafting a block (sample_drafts), same counter and key


def philox4x32_10(counter: np.ndarray, key: np.ndarray) -> np.ndarray:
    """Philox4x32 with 10 rounds [SC11].

    ``counter``: uint32 array [..., 4]; ``key``: uint32 array [..., 2]
    (broadcast against ``counter``). Returns uint32 [..., 4].

    One round maps (c0, c1, c2, c3) with key (k0, k1) to
    (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0)),
    where hi/lo are the upper/lower 32 bits of the 64-bit product. Round r
    (r = 0..9) uses the key (k0 + r*W0, k1 + r*W1) mod 2^32.
    """
    counter = np.asarray(counter, dtype=np.uint32)
    key = np.asarray(key, dtype=np.uint32)
    c0 = counter[..., 0].astype(np.uint64)
    c1 = counter[..., 1].astype(np.uint64)
    c2 = counter[..., 2].astype(np.uint64)
    c3 = counter[..., 3].astype(np.uint64)
    k0 = np.broadcast_to(key[..., 0].astype(np.uint64), c0.shape).copy()
    k1 = np.broadcast_to(key[..., 1].astype(np.uint64), c0.shape).copy()
    for _ in range(10):
        prod0 = _PHILOX_M0 * c0
        prod1 = _PHILOX_M1 * c2
        hi0, lo0 = prod0 >> np.uint64(32), prod0 & _MASK32
        hi1, lo1 = prod1 >> np.uint64(32), prod1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
        k0 = (k0 + _PHILOX_W0) & _MASK32
        k1 = (k1 + _PHILOX_W1) & _MASK32
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def word_to_uniform(word: np.ndarray) -> np.ndarray:
    """u = (word >> 8) * 2^-24, a float64 in {0, 2^-24, ..., 1 - 2^-24}."""
    w = np.asarray(word, dtype=np.uint32) >> np.uint32(8)
    return w.astype(np.float64) * 2.0**-24


def uniforms_for_block(B: int, K: int, seed: int, step: int):
    """Uniforms of one verify call (reading 2).

    Returns ``(u_acc [B, K], u_smp [B, K+1])`` as float64. Counter of
    (sequence b, position i) = (b, i, step lo, step hi); key = (seed lo,
    seed hi). ``u_acc[b, i]`` is word 0 of that block and ``u_smp[b, i]`` is
    word 1.
    """
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    step = int(step) & 0xFFFFFFFFFFFFFFFF
    bb, ii = np.meshgrid(np.arange(B, dtype=np.uint64),
                         np.arange(K + 1, dtype=np.uint64), indexing="ij")
    ctr = np.empty((B, K + 1, 4), dtype=np.uint32)
    ctr[..., 0] = bb.astype(np.uint32)
    ctr[..., 1] = ii.astype(np.uint32)
    ctr[..., 2] = np.uint32(step & 0xFFFFFFFF)
    ctr[..., 3] = np.uint32(step >> 32)
    key = np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint32)
    words = philox4x32_10(ctr, key)
    u_acc = word_to_uniform(words[:, :K, PHILOX_WORD_ACCEPT])
    u_smp = word_to_uniform(words[:, :, PHILOX_WORD_SAMPLE])
    return u_acc, u_smp


# --------------------------------------------------------------------------
# Softmax over the vocabulary (temperature 1)
# --------------------------------------------------------------------------


def softmax_rows(logits: np.ndarray):
    """Row softmax in float64 along the last axis.

    Returns ``(probs, lse)`` with probs = exp(l - m) / Z, Z = sum exp(l - m),
    m = max l, lse = m + log Z. Entries equal to -inf get probability 0.
    """
    l = np.asarray(logits, dtype=np.float64)
    m = np.max(l, axis=-1, keepdims=True)
    e = np.exp(l - m)
    Z = np.sum(e, axis=-1, keepdims=True)
    return e / Z, (m + np.log(Z))[..., 0]


# --------------------------------------------------------------------------
# Verification step of the linear Psi-Spec sampler
# --------------------------------------------------------------------------


def _inverse_cdf(weights: np.ndarray, u: np.ndarray):
    """Inverse-CDF draw per row (reading 4).

    ``weights`` [N, V] are non-negative, unnormalised; ``u`` [N] in [0, 1).
    Returns (index [N], C_prev [N], C_at [N], threshold [N], total [N]) where
    C is the running sum in index order, threshold = u * C_{V-1}, the index
    is the smallest v with C_v > threshold, C_prev = C_{v-1} (0 for v = 0)
    and C_at = C_v. The boundaries let a caller measure how close the draw
    was to a neighbouring token.
    """
    C = np.cumsum(weights, axis=1)
    total = C[:, -1]
    t = u * total
    idx = np.sum(C <= t[:, None], axis=1)
    V = weights.shape[1]
    over = idx >= V
    if np.any(over):
        pos = weights[over] > 0
        last = V - 1 - np.argmax(pos[:, ::-1], axis=1)
        idx = idx.copy()
        idx[over] = last
    rows = np.arange(weights.shape[0])
    C_at = C[rows, idx]
    C_prev = np.where(idx > 0, C[rows, np.maximum(idx - 1, 0)], 0.0)
    return idx, C_prev, C_at, t, total


def verify_block_u(p_logits, q_logits, draft_tokens, u_acc, u_smp):
    """Verify one drafted block per sequence, uniforms given explicitly.

    Arguments (any float dtype; widened to float64):
      p_logits     [B, K+1, V]  verifier (AR) logits; row K is the bonus row
      q_logits     [B, K, V]    draft logits
      draft_tokens [B, K]       drafted ids x_i
      u_acc        [B, K]       accept uniforms u_i in [0, 1)
      u_smp        [B, K+1]     sampling uniforms u'_i in [0, 1)

    Steps, for each sequence b:
      1. p_i = softmax(p_logits[b, i]), q_i = softmax(q_logits[b, i]).
      2. accept_i = u_i * q_i(x_i) < p_i(x_i)                          [SD]
      3. n = index of the first rejected position, K if none.   [READER]
      4. n < K: weights w(v) = max(0, p_n(v) - q_n(v)) (p_n if that is
         all zero); n = K: w = p_K (bonus).                 [SD], [READER]
      5. y = inverse-CDF draw from w with u'_n.
      6. out[0..n-1] = x[0..n-1], out[n] = y, out[n+1..K] = -1.

    Returns a dict with int32 ``out_tokens`` [B, K+1], ``accepted_len`` [B]
    and float64 diagnostics: ``p_at_draft`` / ``q_at_draft`` [B, K],
    ``row_lse`` [B, 2K+1] (p rows 0..K, then q rows 0..K-1), ``ratio``
    [B, K] = p/q at the drafts (inf where q = 0), ``accept`` [B, K] bool,
    and the draw's CDF boundaries ``cdf_prev``, ``cdf_at``, ``cdf_t``,
    ``cdf_total`` [B] (reading 4), with ``cdf_qres`` [B] = the q mass on the
    residual's support, sum of q_n(v) over v with p_n(v) > q_n(v) (0 when the
    draw uses a p row): a diagnostic for comparisons, not part of the method.
    """
    p_logits = np.asarray(p_logits, dtype=np.float64)
    q_logits = np.asarray(q_logits, dtype=np.float64)
    x = np.asarray(draft_tokens).astype(np.int64)
    u_acc = np.asarray(u_acc, dtype=np.float64)
    u_smp = np.asarray(u_smp, dtype=np.float64)
    B, K1, V = p_logits.shape
    K = K1 - 1
    if q_logits.shape != (B, K, V) or x.shape != (B, K):
        raise ValueError("shape mismatch: p [B,K+1,V], q [B,K,V], drafts [B,K]")

    P, lse_p = softmax_rows(p_logits)
    Q, lse_q = softmax_rows(q_logits)

    valid = np.all((x >= 0) & (x < V), axis=1)
    xc = np.clip(x, 0, V - 1)
    p_x = np.take_along_axis(P[:, :K, :], xc[:, :, None], axis=2)[:, :, 0]
    q_x = np.take_along_axis(Q, xc[:, :, None], axis=2)[:, :, 0]

    accept = u_acc * q_x < p_x
    rejected = ~accept
    n = np.where(rejected.any(axis=1), np.argmax(rejected, axis=1), K)

    rows = np.arange(B)
    n_row = np.minimum(n, K - 1)
    resid = np.maximum(0.0, P[rows, n_row, :] - Q[rows, n_row, :])
    resid_empty = resid.sum(axis=1) == 0.0
    use_p_row = np.where(n == K, K, n)
    weights = np.where(((n == K) | resid_empty)[:, None], P[rows, use_p_row, :], resid)
    y, c_prev, c_at, c_t, c_tot = _inverse_cdf(weights, u_smp[rows, n])
    p_n, q_n = P[rows, n_row, :], Q[rows, n_row, :]
    q_res = np.where((n < K) & ~resid_empty, np.sum(np.where(p_n > q_n, q_n, 0.0), axis=1), 0.0)

    out = np.full((B, K + 1), -1, dtype=np.int64)
    cols = np.arange(K + 1)[None, :]
    out = np.where(cols < n[:, None], np.concatenate([x, np.zeros((B, 1), np.int64)], axis=1), out)
    out[rows, n] = y
    acc_len = n.astype(np.int64)
    out[~valid, :] = -1
    acc_len[~valid] = -1

    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(q_x > 0, p_x / q_x, np.inf)

    return {
        "out_tokens": out.astype(np.int32),
        "accepted_len": acc_len.astype(np.int32),
        "p_at_draft": p_x,
        "q_at_draft": q_x,
        "row_lse": np.concatenate([lse_p, lse_q], axis=1),
        "ratio": ratio,
        "u_acc": u_acc,
        "u_smp": u_smp[rows, n],
        "accept": accept,
        "valid": valid,
        "cdf_prev": c_prev,
        "cdf_at": c_at,
        "cdf_t": c_t,
        "cdf_total": c_tot,
        "cdf_qres": q_res,
    }


def verify_block(p_logits, q_logits, draft_tokens, seed: int, step: int):
    """``verify_block_u`` with the Philox uniforms of (seed, step) (reading 2)."""
    p_logits = np.asarray(p_logits)
    B, K1, _ = p_logits.shape
    u_acc, u_smp = uniforms_for_block(B, K1 - 1, seed, step)
    return verify_block_u(p_logits, q_logits, draft_tokens, u_acc, u_smp)


# --------------------------------------------------------------------------
# Dual-pathway linear
# --------------------------------------------------------------------------


def dualpath_linear(x, W, A, Bm, scale: float, round_t_to_bf16: bool, gate=None):
    """Dual-pathway linear of a diffusion-augmented layer, float64.

    x [M, d_in], W [d_out, d_in] (frozen AR weight, ``nn.Linear`` layout),
    A [r, d_in] (LoRA down), Bm [d_out, r] (LoRA up), scale = alpha / r.

      y_AR    = x W^T                      (verification pathway)
      T       = scale * x A^T              (rounded to bf16 if asked, reading 8)
      y_draft = y_AR + T Bm^T              (drafting pathway, theta_AR + theta_Delta)

    gate [M] (optional, nonzero = adapter on): the gated LoRA of the reader
    page, "The Psi-Speculative Sampler" (logits of token 1 of a draft block
    use the AR weights alone, tokens 2..B the gated LoRA-augmented weights) and
    "Supplementary Details" (the first position's clean-token distribution uses
    theta_AR only). A row with gate 0 has T = 0, so its y_draft is its y_AR.

    Returns (y_AR [M, d_out], y_draft [M, d_out], T [M, r]).
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bm = np.asarray(Bm, dtype=np.float64)
    y_ar = x @ W.T
    T = float(scale) * (x @ A.T)
    if round_t_to_bf16:
        T = round_to_bf16(T)
    if gate is not None:
        on = np.asarray(gate).reshape(-1) != 0
        T = np.where(on[:, None], T, 0.0)
    y_draft = y_ar + T @ Bm.T
    return y_ar, y_draft, T


# --------------------------------------------------------------------------
# Drafting: the linear sampler's proposal
# --------------------------------------------------------------------------


def draft_uniforms(B: int, K: int, seed: int, step: int):
    """Uniforms of a draft call: word 2 of the Philox block of (sequence b,
    position i) with the counter and key of uniforms_for_block; [B, K]."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    step = int(step) & 0xFFFFFFFFFFFFFFFF
    bb, ii = np.meshgrid(np.arange(B, dtype=np.uint64), np.arange(K, dtype=np.uint64),
                         indexing="ij")
    ctr = np.empty((B, K, 4), dtype=np.uint32)
    ctr[..., 0] = bb.astype(np.uint32)
    ctr[..., 1] = ii.astype(np.uint32)
    ctr[..., 2] = np.uint32(step & 0xFFFFFFFF)
    ctr[..., 3] = np.uint32(step >> 32)
    key = np.array([seed & 0xFFFFFFFF, seed >> 32], dtype=np.uint32)
    return word_to_uniform(philox4x32_10(ctr, key)[..., PHILOX_WORD_DRAFT])


def sample_drafts_u(q_logits, u):
    """Drafted ids of the linear sampler for given uniforms u [B, K].

    The linear sampler draws the block's tokens in parallel, each from its
    own marginal (reader page, "The Psi-Speculative Sampler": sample a
    candidate set from the joint proposal, linear or tree-based; the summary
    page's "Psi-Speculative Sampler"): x_{b,i} ~ softmax(q_{b,i}), here by the
    inverse CDF of reading 4 over exp(q - max) in index order. A row with no
    finite logit has no distribution: its id is -1.

    Returns (ids [B, K] int32, details) where details holds the CDF
    boundaries of each draw (for near-tie accounting).
    """
    q = np.asarray(q_logits, dtype=np.float64)
    B, K, V = q.shape
    rows = q.reshape(B * K, V)
    finite = np.isfinite(rows).any(axis=1)
    m = np.where(finite, np.max(np.where(np.isfinite(rows), rows, -np.inf), axis=1), 0.0)
    w = np.where(np.isfinite(rows), np.exp(rows - m[:, None]), 0.0)
    idx, c_prev, c_at, t, total = _inverse_cdf(w, np.asarray(u, dtype=np.float64).reshape(-1))
    idx = np.where(finite, idx, -1).astype(np.int32)
    # sqrt(sum of squared weights): the scale at which uncorrelated per-token
    # relative errors of a float32 implementation move the CDF (diagnostic,
    # for near-tie accounting only)
    spread = np.sqrt(np.sum(w * w, axis=1))
    details = {"c_prev": c_prev.reshape(B, K), "c_at": c_at.reshape(B, K),
               "threshold": t.reshape(B, K), "total": total.reshape(B, K),
               "spread": spread.reshape(B, K)}
    return idx.reshape(B, K), details


def sample_drafts(q_logits, seed: int, step: int):
    """Drafted ids for one block: sample_drafts_u with draft_uniforms."""
    q = np.asarray(q_logits)
    return sample_drafts_u(q, draft_uniforms(q.shape[0], q.shape[1], seed, step))


# --------------------------------------------------------------------------
# The LM head feeding the verifier (the fused row): row statistics per column
# tile and the verifier on the LM head's row layout
# --------------------------------------------------------------------------


def row_stat_partials(y, tile: int = 256):
    """Softmax partials of each row of y [M, N] per column tile, float64.

    Tile t covers columns [t*tile, (t+1)*tile). Its partial is
    (m, z) = (max(y) * log2(e), sum of 2^(y * log2(e) - m)) over the tile's
    finite entries, (-inf, 0) when it has none. Merging the partials of a row
    gives its normaliser: log Z = ln 2 * (M + log2 sum_t z_t 2^(m_t - M)),
    M = max_t m_t. Returns an array [M, T, 2].
    """
    y = np.asarray(y, dtype=np.float64)
    M, N = y.shape
    T = (N + tile - 1) // tile
    out = np.empty((M, T, 2))
    log2e = 1.0 / np.log(2.0)
    for t in range(T):
        blk = y[:, t * tile:(t + 1) * tile] * log2e
        fin = np.isfinite(blk)
        m = np.where(fin, blk, -np.inf).max(axis=1)
        has = np.isfinite(m)
        ref = np.where(has, m, 0.0)
        z = np.where(fin, np.exp2(np.where(fin, blk, 0.0) - ref[:, None]), 0.0).sum(axis=1)
        out[:, t, 0] = m
        out[:, t, 1] = np.where(has, z, 0.0)
    return out


def merge_row_stats(partials):
    """Natural-log normaliser of each row from its [T, 2] partials."""
    p = np.asarray(partials, dtype=np.float64)
    m, z = p[..., 0], p[..., 1]
    top = m.max(axis=-1)
    safe = np.where(np.isfinite(top), top, 0.0)
    w = np.where(np.isfinite(m), z * np.exp2(m - safe[..., None]), 0.0).sum(axis=-1)
    ok = np.isfinite(top)
    return np.where(ok, (top + np.log2(np.where(ok, w, 1.0))) * np.log(2.0), -np.inf)


def verify_block_head(y_ar, y_draft, draft_tokens, seed: int, step: int):
    """The verifier on the LM head's outputs, as the fused entry reads them.

    y_ar, y_draft [B*(K+1), V]: one block of K+1 rows per sequence. The
    verifier's p is the block's K+1 AR rows; q_i is the block's draft row i
    for i < K (the bonus position's draft row is not a draft distribution of
    any drafted token). Then ``verify_block``.
    """
    x = np.asarray(draft_tokens)
    B, K = x.shape
    y_ar = np.asarray(y_ar, dtype=np.float64)
    V = y_ar.shape[-1]
    p = y_ar.reshape(B, K + 1, V)
    q = np.asarray(y_draft, dtype=np.float64).reshape(B, K + 1, V)[:, :K]
    return verify_block(p, q, x, seed=seed, step=step)
