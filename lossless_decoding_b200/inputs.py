"""Seeded synthetic inputs for the dual-path linear and the block verifier.

This module only draws random inputs; it holds none of the method's
arithmetic (no softmax, no accept rule, no GEMM), so both the CUDA path's
tests and the float64 oracle can be fed from it without sharing any logic.
The shapes and distributions stand in for the paper's Qwen3-8B setting
("Unlocking Lossless Speedups in LLMs via Discrete Diffusion", Empirical
Results: Qwen3-8B augmented with rank-128 LoRA diffusion weights; 1K/8K
throughput test at batch 1 and 64). No dataset or checkpoint is used.

Every generator takes a ``seed`` and a ``device``; on a given device the
output is a pure function of the arguments. CPU and CUDA generators produce
different streams for the same seed.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}

# Qwen3-8B-shaped projection set of one decoder layer (d_in, d_out):
# q and o 4096->4096, k and v 4096->1024, gate and up 4096->12288,
# down 12288->4096.
QWEN3_8B_PROJECTIONS = (
    ("q", 4096, 4096),
    ("k", 4096, 1024),
    ("v", 4096, 1024),
    ("o", 4096, 4096),
    ("gate", 4096, 12288),
    ("up", 4096, 12288),
    ("down", 12288, 4096),
)
QWEN3_8B_HIDDEN = 4096
QWEN3_8B_VOCAB = 151936
QWEN3_8B_LAYERS = 36


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _gumbel(shape, g: torch.Generator, device) -> torch.Tensor:
    """Standard Gumbel(0, 1) noise, float32."""
    u = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    u = u.clamp_(min=1e-20, max=1.0 - 1e-7)
    return -torch.log(-torch.log(u))


@dataclass
class VerifyInputs:
    p_logits: torch.Tensor      # [B, K+1, V]
    q_logits: torch.Tensor      # [B, K, V]
    draft_tokens: torch.Tensor  # [B, K] int32


def verify_inputs(B: int, K: int, V: int, dtype: str = "bf16", dist: str = "normal",
                  p_std: float = 2.0, sigma: float = 0.5, boost_count: int = 20,
                  boost: float = 8.0, seed: int = 0, device="cpu",
                  drafts: str = "sample") -> VerifyInputs:
    """Verifier logits and drafted ids.

    dist = "normal": AR logits ~ N(0, p_std^2).
    dist = "gumbel": AR logits ~ Gumbel(0, 1) with ``boost_count`` random
                     tokens per row raised by ``boost`` (heavy top-k mass).
    Draft logits q = AR logits (rows 0..K-1) + N(0, sigma^2), both stored in
    ``dtype``. ``drafts = "sample"`` draws each x_i from the categorical of
    the stored q row by the Gumbel-max trick; ``drafts = "uniform"`` draws
    ids uniformly from [0, V).
    """
    g = _gen(seed, device)
    shape = (B, K + 1, V)
    if dist == "normal":
        p = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * p_std
    elif dist == "gumbel":
        p = _gumbel(shape, g, device)
        if boost_count > 0 and V > 0:
            idx = torch.randint(0, V, (B, K + 1, min(boost_count, V)), generator=g, device=device)
            p.scatter_add_(2, idx, torch.full(idx.shape, float(boost), device=device))
    else:
        raise ValueError(f"unknown dist {dist!r}")
    q = p[:, :K, :] + sigma * torch.randn((B, K, V), generator=g, device=device,
                                          dtype=torch.float32)
    tdt = DTYPES[dtype]
    p_t = p.to(tdt).contiguous()
    q_t = q.to(tdt).contiguous()
    del p, q
    if drafts == "sample":
        x = torch.empty((B, K), dtype=torch.int32, device=device)
        for b in range(B):  # bounded memory for large B*K*V
            noisy = q_t[b].float() + _gumbel((K, V), g, device)
            x[b] = torch.argmax(noisy, dim=1).to(torch.int32)
    elif drafts == "uniform":
        x = torch.randint(0, V, (B, K), generator=g, device=device, dtype=torch.int32)
    else:
        raise ValueError(f"unknown drafts {drafts!r}")
    return VerifyInputs(p_t, q_t, x)


@dataclass
class DualPathInputs:
    x: torch.Tensor   # [M, d_in]
    W: torch.Tensor   # [d_out, d_in]
    A: torch.Tensor   # [r, d_in]
    Bm: torch.Tensor  # [d_out, r]
    scale: float      # alpha / r


def dualpath_inputs(M: int, d_in: int, d_out: int, r: int, alpha: float,
                    dtype: str = "bf16", w_std: float = 0.02, a_std: float = 0.02,
                    b_std: float = 0.02, x_std: float = 1.0, seed: int = 0,
                    device="cpu") -> DualPathInputs:
    """Activations and frozen/LoRA weights of one dual-path linear."""
    g = _gen(seed, device)
    tdt = DTYPES[dtype]

    def draw(shape, std):
        return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(tdt)

    x = draw((M, d_in), x_std)
    W = draw((d_out, d_in), w_std)
    A = draw((r, d_in), a_std)
    Bm = draw((d_out, r), b_std)
    return DualPathInputs(x, W, A, Bm, float(alpha) / float(r))


# --------------------------------------------------------------------------
# Named workloads. Sizes follow the paper's 8B setting; the recipes are the
# ones the tests and the benchmark draw from.
# --------------------------------------------------------------------------

WORKLOADS = {
    "tiny": dict(B=1, K=8, V=4096, dtype="f32", dist="normal", p_std=2.0, sigma=0.5,
                 M=8, d_in=512, d_out=512, r=16, alpha=32.0, w_std=0.02, a_std=0.02,
                 b_std=0.01),
    "qwen3_8b_b1": dict(B=1, K=16, V=QWEN3_8B_VOCAB, dtype="bf16", sigma=1.0,
                        d_in=QWEN3_8B_HIDDEN, r=128, alpha=256.0),
    "batched_decode_b64_k16": dict(B=64, K=16, V=QWEN3_8B_VOCAB, dtype="bf16",
                                   dist="normal", p_std=2.0, sigma=1.0, r=128,
                                   alpha=256.0),
}
