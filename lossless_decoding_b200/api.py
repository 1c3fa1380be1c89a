"""PyTorch-facing binding of the Uno C ABI (argument marshalling only).

Every step of the computation runs in libuno.so's sm_100a kernels; this
module checks tensor devices, dtypes and shapes, allocates outputs and
workspaces through PyTorch, and passes raw pointers and the current CUDA
stream to the C entry points of the same names.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from ._lib import UNO_BF16, UNO_F32, UnoError, lib

_DT = {torch.bfloat16: UNO_BF16, torch.float32: UNO_F32}


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32") from None


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_cuda(*ts: Optional[torch.Tensor]) -> torch.device:
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous (row-major, no padding)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must live on the same device")
    return dev


def _stream_handle(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


class _Workspaces:
    """Grow-only device scratch buffers, one per (device, purpose).

    The kernels do not depend on a workspace's previous contents. Calls that
    use one cached workspace are ordered on the current stream of the caller.
    """

    def __init__(self):
        self._bufs: dict = {}

    def get(self, device: torch.device, purpose: str, nbytes: int) -> torch.Tensor:
        key = (device.index, purpose)
        buf = self._bufs.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
            self._bufs[key] = buf
        return buf


_ws = _Workspaces()


# ---------------------------------------------------------------------------
# block verifier
# ---------------------------------------------------------------------------


@dataclass
class VerifyResult:
    out_tokens: torch.Tensor            # [B, K+1] int32, -1 padded
    accepted_len: torch.Tensor          # [B] int32 (-1 marks an invalid draft id)
    p_at_draft: Optional[torch.Tensor]  # [B, K] float32
    q_at_draft: Optional[torch.Tensor]  # [B, K] float32
    row_lse: Optional[torch.Tensor]     # [B, 2K+1] float32


def verify_workspace_bytes(B: int, K: int, V: int, dtype: torch.dtype) -> int:
    return int(lib.uno_verify_workspace_bytes(B, K, V, _DT[dtype]))


def verify_block(p_logits: torch.Tensor, q_logits: torch.Tensor, draft_tokens: torch.Tensor,
                 seed: int, step: int, *, want_probs: bool = False, want_lse: bool = False,
                 out: Optional[VerifyResult] = None,
                 workspace: Optional[torch.Tensor] = None) -> VerifyResult:
    """Verify one drafted block per sequence (see ``uno_verify_block`` in uno.h).

    p_logits [B, K+1, V] and q_logits [B, K, V] (bfloat16 or float32, same
    dtype), draft_tokens [B, K] int32. Runs asynchronously on the current
    stream.
    """
    if p_logits.dim() != 3 or q_logits.dim() != 3 or draft_tokens.dim() != 2:
        raise ValueError("expected p [B,K+1,V], q [B,K,V], drafts [B,K]")
    B, K1, V = p_logits.shape
    K = K1 - 1
    if tuple(q_logits.shape) != (B, K, V) or tuple(draft_tokens.shape) != (B, K):
        raise ValueError("shape mismatch: p [B,K+1,V], q [B,K,V], drafts [B,K]")
    if q_logits.dtype != p_logits.dtype:
        raise TypeError("p_logits and q_logits must share a dtype")
    if draft_tokens.dtype != torch.int32:
        raise TypeError("draft_tokens must be int32")
    dt = _dtype_code(p_logits)
    dev = _check_cuda(p_logits, q_logits, draft_tokens)
    if out is None:
        out = VerifyResult(
            torch.empty((B, K + 1), dtype=torch.int32, device=dev),
            torch.empty((B,), dtype=torch.int32, device=dev),
            torch.empty((B, K), dtype=torch.float32, device=dev) if want_probs else None,
            torch.empty((B, K), dtype=torch.float32, device=dev) if want_probs else None,
            torch.empty((B, 2 * K + 1), dtype=torch.float32, device=dev) if want_lse else None,
        )
    _check_cuda(out.out_tokens, out.accepted_len, out.p_at_draft, out.q_at_draft, out.row_lse)
    need = int(lib.uno_verify_workspace_bytes(B, K, V, dt))
    ws = workspace if workspace is not None else _ws.get(dev, "verify", need)
    st = lib.uno_verify_block(
        _ptr(p_logits), _ptr(q_logits), _ptr(draft_tokens), B, K, V, dt,
        ctypes.c_uint64(int(seed) & (2**64 - 1)), ctypes.c_uint64(int(step) & (2**64 - 1)),
        _ptr(out.out_tokens), _ptr(out.accepted_len), _ptr(out.p_at_draft),
        _ptr(out.q_at_draft), _ptr(out.row_lse), _ptr(ws), ws.numel(), _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_verify_block")
    return out


def verify_block_noalloc(p_logits: torch.Tensor, q_logits: torch.Tensor,
                         draft_tokens: torch.Tensor, seed: int, step: int, *,
                         out: VerifyResult) -> VerifyResult:
    """``uno_verify_block_noalloc``: the verifier without a workspace.

    For callers that cannot allocate device memory at call time: the library
    uses its own fixed 4 MiB scratch array and the caller supplies every
    output buffer in ``out``. Calls on one device share that scratch, so keep
    them on one stream. Problems needing more than 4 MiB of scratch raise
    UnoError (UNO_ERR_SIZE).
    """
    B, K1, V = p_logits.shape
    K = K1 - 1
    dt = _dtype_code(p_logits)
    dev = _check_cuda(p_logits, q_logits, draft_tokens, out.out_tokens, out.accepted_len,
                      out.p_at_draft, out.q_at_draft, out.row_lse)
    st = lib.uno_verify_block_noalloc(
        _ptr(p_logits), _ptr(q_logits), _ptr(draft_tokens), B, K, V, dt,
        ctypes.c_uint64(int(seed) & (2**64 - 1)), ctypes.c_uint64(int(step) & (2**64 - 1)),
        _ptr(out.out_tokens), _ptr(out.accepted_len), _ptr(out.p_at_draft),
        _ptr(out.q_at_draft), _ptr(out.row_lse), _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_verify_block_noalloc")
    return out


# ---------------------------------------------------------------------------
# dual-pathway linear
# ---------------------------------------------------------------------------


def dualpath_workspace_bytes(M: int, d_in: int, d_out: int, r: int, dtype: torch.dtype) -> int:
    return int(lib.uno_dualpath_workspace_bytes(M, d_in, d_out, r, _DT[dtype]))


def _gate_arg(gate: Optional[torch.Tensor], M: int, dev) -> Optional[int]:
    if gate is None:
        return None
    if gate.dtype not in (torch.uint8, torch.bool) or gate.numel() != M or not gate.is_contiguous():
        raise ValueError("gate must be a contiguous uint8/bool tensor with one entry per row")
    _check_cuda(gate)
    if gate.device != dev:
        raise ValueError("gate must live on the same device")
    return gate.data_ptr()


def dualpath_linear(x: torch.Tensor, W: torch.Tensor, A: torch.Tensor, Bm: torch.Tensor,
                    scale: float, *, want_ar: bool = True, want_draft: bool = True,
                    y_ar: Optional[torch.Tensor] = None, y_draft: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None,
                    gate: Optional[torch.Tensor] = None):
    """y_ar = x W^T and y_draft = y_ar + scale (x A^T) Bm^T in one pass over W.

    x [M, d_in], W [d_out, d_in], A [r, d_in], Bm [d_out, r], all bfloat16 or
    all float32. gate [M] (uint8/bool, optional): rows with gate 0 get no
    adapter (their y_draft equals y_ar). Returns (y_ar, y_draft); an output not
    wanted is None.
    """
    if x.dim() != 2 or W.dim() != 2 or A.dim() != 2 or Bm.dim() != 2:
        raise ValueError("expected 2-D x, W, A, Bm")
    M, d_in = x.shape
    d_out = W.shape[0]
    r = A.shape[0]
    if W.shape[1] != d_in or A.shape[1] != d_in or tuple(Bm.shape) != (d_out, r):
        raise ValueError("shape mismatch: x [M,d_in], W [d_out,d_in], A [r,d_in], Bm [d_out,r]")
    if not (x.dtype == W.dtype == A.dtype == Bm.dtype):
        raise TypeError("x, W, A and Bm must share a dtype")
    dt = _dtype_code(x)
    dev = _check_cuda(x, W, A, Bm)
    if want_ar and y_ar is None:
        y_ar = torch.empty((M, d_out), dtype=x.dtype, device=dev)
    if want_draft and y_draft is None:
        y_draft = torch.empty((M, d_out), dtype=x.dtype, device=dev)
    if not want_ar:
        y_ar = None
    if not want_draft:
        y_draft = None
    _check_cuda(y_ar, y_draft)
    need = int(lib.uno_dualpath_workspace_bytes(M, d_in, d_out, r, dt))
    ws = workspace if workspace is not None else _ws.get(dev, "dualpath", need)
    if gate is None:
        st = lib.uno_dualpath_linear(_ptr(x), _ptr(W), _ptr(A), _ptr(Bm), ctypes.c_float(scale),
                                     _ptr(y_ar), _ptr(y_draft), M, d_in, d_out, r, dt, _ptr(ws),
                                     ws.numel(), _stream_handle(dev))
    else:
        st = lib.uno_dualpath_linear_gated(_ptr(x), _ptr(W), _ptr(A), _ptr(Bm),
                                           ctypes.c_float(scale), _gate_arg(gate, M, dev),
                                           _ptr(y_ar), _ptr(y_draft), M, d_in, d_out, r, dt,
                                           _ptr(ws), ws.numel(), _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_dualpath_linear")
    return y_ar, y_draft


def dualpath_stats_tiles(M: int, d_out: int) -> int:
    """Softmax partials per row written by ``dualpath_linear_stats``: one per
    256-column tile when M > 256, one per CTA (148) when M <= 256, 0 for an
    empty problem."""
    return int(lib.uno_dualpath_stats_tiles(M, d_out))


def dualpath_linear_stats(x: torch.Tensor, W: torch.Tensor, A: torch.Tensor, Bm: torch.Tensor,
                          scale: float, *, gate: Optional[torch.Tensor] = None,
                          y_ar: Optional[torch.Tensor] = None,
                          y_draft: Optional[torch.Tensor] = None,
                          stats_ar: Optional[torch.Tensor] = None,
                          stats_draft: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None):
    """The LM head: ``dualpath_linear`` (both outputs) that also writes each
    output row's softmax partials, float32 [M, T, 2] as (max * log2 e, sum
    of 2^(x log2 e - that)), each over a part of the row (T =
    ``dualpath_stats_tiles``; an empty part is (-inf, 0)). Returns (y_ar,
    y_draft, stats_ar, stats_draft)."""
    if x.dim() != 2 or W.dim() != 2 or A.dim() != 2 or Bm.dim() != 2:
        raise ValueError("expected 2-D x, W, A, Bm")
    M, d_in = x.shape
    d_out = W.shape[0]
    r = A.shape[0]
    if W.shape[1] != d_in or A.shape[1] != d_in or tuple(Bm.shape) != (d_out, r):
        raise ValueError("shape mismatch: x [M,d_in], W [d_out,d_in], A [r,d_in], Bm [d_out,r]")
    if not (x.dtype == W.dtype == A.dtype == Bm.dtype):
        raise TypeError("x, W, A and Bm must share a dtype")
    T = dualpath_stats_tiles(M, d_out)
    if T == 0:
        raise ValueError("row statistics need M >= 1 and d_out >= 1")
    dt = _dtype_code(x)
    dev = _check_cuda(x, W, A, Bm)
    if y_ar is None:
        y_ar = torch.empty((M, d_out), dtype=x.dtype, device=dev)
    if y_draft is None:
        y_draft = torch.empty((M, d_out), dtype=x.dtype, device=dev)
    if stats_ar is None:
        stats_ar = torch.empty((M, T, 2), dtype=torch.float32, device=dev)
    if stats_draft is None:
        stats_draft = torch.empty((M, T, 2), dtype=torch.float32, device=dev)
    for t in (stats_ar, stats_draft):
        if t.dtype != torch.float32 or tuple(t.shape) != (M, T, 2):
            raise ValueError(f"stats must be float32 [{M}, {T}, 2]")
    _check_cuda(y_ar, y_draft, stats_ar, stats_draft)
    need = int(lib.uno_dualpath_workspace_bytes(M, d_in, d_out, r, dt))
    ws = workspace if workspace is not None else _ws.get(dev, "dualpath", need)
    st = lib.uno_dualpath_linear_stats(_ptr(x), _ptr(W), _ptr(A), _ptr(Bm), ctypes.c_float(scale),
                                       None if gate is None else _gate_arg(gate, M, dev),
                                       _ptr(y_ar), _ptr(y_draft), _ptr(stats_ar),
                                       _ptr(stats_draft), M, d_in, d_out, r, dt, _ptr(ws),
                                       ws.numel(), _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_dualpath_linear_stats")
    return y_ar, y_draft, stats_ar, stats_draft


def verify_block_head(y_ar: torch.Tensor, y_draft: torch.Tensor, stats_ar: torch.Tensor,
                      stats_draft: torch.Tensor, draft_tokens: torch.Tensor, seed: int,
                      step: int, *, want_probs: bool = False, want_lse: bool = False,
                      out: Optional[VerifyResult] = None,
                      workspace: Optional[torch.Tensor] = None) -> VerifyResult:
    """Verify from the LM head's outputs and row statistics: y_ar, y_draft
    [B*(K+1), V] (or [B, K+1, V]) with p = y_ar rows and q_i = y_draft row
    b*(K+1)+i for i < K; stats from ``dualpath_linear_stats``."""
    B, K = draft_tokens.shape
    V = y_ar.shape[-1]
    if y_ar.numel() != B * (K + 1) * V or y_draft.shape != y_ar.shape:
        raise ValueError("y_ar and y_draft must hold B*(K+1) rows of V logits")
    if stats_ar.dim() != 3 or stats_ar.shape[0] != B * (K + 1) or stats_ar.shape[2] != 2 \
            or stats_draft.shape != stats_ar.shape:
        raise ValueError("stats must be float32 [B*(K+1), T, 2]")
    if draft_tokens.dtype != torch.int32:
        raise TypeError("draft_tokens must be int32")
    T = stats_ar.shape[1]
    dt = _dtype_code(y_ar)
    dev = _check_cuda(y_ar, y_draft, stats_ar, stats_draft, draft_tokens)
    if out is None:
        out = VerifyResult(
            torch.empty((B, K + 1), dtype=torch.int32, device=dev),
            torch.empty((B,), dtype=torch.int32, device=dev),
            torch.empty((B, K), dtype=torch.float32, device=dev) if want_probs else None,
            torch.empty((B, K), dtype=torch.float32, device=dev) if want_probs else None,
            torch.empty((B, 2 * K + 1), dtype=torch.float32, device=dev) if want_lse else None,
        )
    _check_cuda(out.out_tokens, out.accepted_len, out.p_at_draft, out.q_at_draft, out.row_lse)
    need = int(lib.uno_verify_workspace_bytes(B, K, V, dt))
    ws = workspace if workspace is not None else _ws.get(dev, "verify", need)
    st = lib.uno_verify_block_head(
        _ptr(y_ar), _ptr(y_draft), _ptr(stats_ar), _ptr(stats_draft), T, _ptr(draft_tokens),
        B, K, V, dt, ctypes.c_uint64(int(seed) & (2**64 - 1)),
        ctypes.c_uint64(int(step) & (2**64 - 1)), _ptr(out.out_tokens), _ptr(out.accepted_len),
        _ptr(out.p_at_draft), _ptr(out.q_at_draft), _ptr(out.row_lse), _ptr(ws), ws.numel(),
        _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_verify_block_head")
    return out


def dualpath_linear_grouped(x: torch.Tensor, Ws, As, Bms, scales, *, want_ar: bool = True,
                            want_draft: bool = True, y_ars=None, y_drafts=None,
                            workspace: Optional[torch.Tensor] = None,
                            gate: Optional[torch.Tensor] = None):
    """Several dual-path projections of the same x in one launch.

    Ws[g] [d_out_g, d_in], As[g] [r, d_in], Bms[g] [d_out_g, r], scales[g];
    1 to 4 projections, one dtype. `want_ar` is one flag or one per
    projection. Returns (y_ars, y_drafts), lists with one entry per projection
    (entries None when not wanted).
    """
    n = len(Ws)
    if not (1 <= n <= 4) or len(As) != n or len(Bms) != n or len(scales) != n:
        raise ValueError("need 1 to 4 projections with one W, A, Bm and scale each")
    if x.dim() != 2:
        raise ValueError("expected 2-D x")
    M, d_in = x.shape
    r = As[0].shape[0]
    d_outs = []
    for W, A, Bm in zip(Ws, As, Bms):
        if W.dim() != 2 or A.dim() != 2 or Bm.dim() != 2:
            raise ValueError("expected 2-D W, A, Bm")
        d_out = W.shape[0]
        if W.shape[1] != d_in or tuple(A.shape) != (r, d_in) or tuple(Bm.shape) != (d_out, r):
            raise ValueError("shape mismatch: x [M,d_in], W [d_out,d_in], A [r,d_in], Bm [d_out,r]")
        if not (x.dtype == W.dtype == A.dtype == Bm.dtype):
            raise TypeError("x, W, A and Bm must share a dtype")
        d_outs.append(d_out)
    dt = _dtype_code(x)
    dev = _check_cuda(x, *Ws, *As, *Bms)
    y_ars = list(y_ars) if y_ars is not None else [None] * n
    y_drafts = list(y_drafts) if y_drafts is not None else [None] * n
    # want_ar may be one flag or one per projection; y_draft is all or none
    wants_ar = list(want_ar) if isinstance(want_ar, (list, tuple)) else [bool(want_ar)] * n
    if len(wants_ar) != n:
        raise ValueError("want_ar: one flag, or one per projection")
    for g in range(n):
        if wants_ar[g] and y_ars[g] is None:
            y_ars[g] = torch.empty((M, d_outs[g]), dtype=x.dtype, device=dev)
        if want_draft and y_drafts[g] is None:
            y_drafts[g] = torch.empty((M, d_outs[g]), dtype=x.dtype, device=dev)
        if not wants_ar[g]:
            y_ars[g] = None
        if not want_draft:
            y_drafts[g] = None
    _check_cuda(*y_ars, *y_drafts)
    c_dout = (ctypes.c_int * n)(*d_outs)
    need = int(lib.uno_dualpath_grouped_workspace_bytes(n, M, d_in, c_dout, r, dt))
    ws = workspace if workspace is not None else _ws.get(dev, "dualpath", need)
    vpa = ctypes.c_void_p * n
    st = lib.uno_dualpath_linear_grouped(
        n, _ptr(x), vpa(*[_ptr(t) for t in Ws]), vpa(*[_ptr(t) for t in As]),
        vpa(*[_ptr(t) for t in Bms]), (ctypes.c_float * n)(*[float(s) for s in scales]),
        _gate_arg(gate, M, dev), vpa(*[_ptr(t) for t in y_ars]), vpa(*[_ptr(t) for t in y_drafts]), M, d_in, c_dout, r,
        dt, _ptr(ws), ws.numel(), _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_dualpath_linear_grouped")
    return y_ars, y_drafts


# ---------------------------------------------------------------------------
# drafting a block
# ---------------------------------------------------------------------------


def sample_drafts(q_logits: torch.Tensor, seed: int, step: int, *,
                  out: Optional[torch.Tensor] = None,
                  num_drafts: Optional[int] = None) -> torch.Tensor:
    """Drafted ids of the linear sampler: out[b, i] ~ softmax(q_logits[b, i]).

    q_logits [B, R, V] bfloat16 or float32 on a CUDA device, contiguous;
    draws rows i < K of each block, K = num_drafts (default R; for example
    R = K + 1 for the LM head's draft-pathway output, whose last row per block
    is then not read). Returns int32 [B, K] (-1 for a row with no finite
    logit). Uniform: Philox word 2 of (b, i, step) under key `seed`, next to
    the verifier's words 0 and 1.
    """
    if q_logits.dim() != 3:
        raise ValueError("q_logits must be [B, R, V]")
    if not q_logits.is_contiguous():
        raise ValueError("q_logits must be contiguous")
    B, R, V = q_logits.shape
    K = R if num_drafts is None else int(num_drafts)
    if not 1 <= K <= R:
        raise ValueError("num_drafts must be in [1, R]")
    dt = _dtype_code(q_logits)
    dev = _check_cuda(q_logits)
    if out is None:
        out = torch.empty((B, K), dtype=torch.int32, device=dev)
    if out.dtype != torch.int32 or tuple(out.shape) != (B, K):
        raise ValueError("out must be int32 [B, K]")
    _check_cuda(out)
    st = lib.uno_sample_drafts_blocks(_ptr(q_logits), B, K, R, V, dt,
                                      ctypes.c_uint64(seed & (2**64 - 1)),
                                      ctypes.c_uint64(step & (2**64 - 1)), _ptr(out),
                                      _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_sample_drafts_blocks")
    return out


# ---------------------------------------------------------------------------
# tree sampler
# ---------------------------------------------------------------------------


@dataclass
class DraftTree:
    """A candidate tree per sequence (as ``uno_tree_draft`` writes it)."""

    topk_ids: torch.Tensor     # [B, D, top_k] int32
    topk_logq: torch.Tensor    # [B, D, top_k] float32
    node_token: torch.Tensor   # [B, N] int32
    node_parent: torch.Tensor  # [B, N] int32
    node_depth: torch.Tensor   # [B, N] int32
    n_nodes: torch.Tensor      # [B] int32
    budget: int


def tree_nodes(depth: int, budget: int) -> int:
    """Node rows N of a tree of `depth` positions and `budget` kept sequences."""
    n = lib.uno_tree_nodes(depth, budget)
    if n <= 0:
        raise ValueError("depth must be in [1, 16] and budget in [1, 64]")
    return n


def tree_draft_workspace_bytes(B: int, D: int, V: int, top_k: int) -> int:
    return int(lib.uno_tree_draft_workspace_bytes(B, D, V, top_k))


def tree_draft(q_logits: torch.Tensor, top_k: int, budget: int, *,
               workspace: Optional[torch.Tensor] = None) -> DraftTree:
    """Top-k candidates of each position and the tree of the `budget` best
    sequences by joint log-probability. q_logits [B, D, V] bf16/f32."""
    if q_logits.dim() != 3:
        raise ValueError("q_logits must be [B, D, V]")
    B, D, V = q_logits.shape
    dt = _dtype_code(q_logits)
    dev = _check_cuda(q_logits)
    N = tree_nodes(D, budget)
    i32 = dict(dtype=torch.int32, device=dev)
    t = DraftTree(torch.empty((B, D, top_k), **i32),
                  torch.empty((B, D, top_k), dtype=torch.float32, device=dev),
                  torch.empty((B, N), **i32), torch.empty((B, N), **i32),
                  torch.empty((B, N), **i32), torch.empty((B,), **i32), budget)
    need = lib.uno_tree_draft_workspace_bytes(B, D, V, top_k)
    if need == 0:
        raise ValueError("sizes out of range for the tree sampler")
    if workspace is None:
        workspace = _ws.get(dev, "tree_draft", need)
    if workspace.dtype != torch.uint8 or workspace.numel() < need:
        raise ValueError(f"workspace must be uint8 with at least {need} bytes")
    _check_cuda(workspace)
    st = lib.uno_tree_draft(_ptr(q_logits), B, D, V, dt, top_k, budget, _ptr(t.topk_ids),
                            _ptr(t.topk_logq), _ptr(t.node_token), _ptr(t.node_parent),
                            _ptr(t.node_depth), _ptr(t.n_nodes), _ptr(workspace), need,
                            _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_tree_draft")
    return t


@dataclass
class TreeResult:
    out_tokens: torch.Tensor    # [B, D+1] int32
    accepted_len: torch.Tensor  # [B] int32
    node_draw: torch.Tensor     # [B, N] int32


def tree_verify(p_logits: torch.Tensor, tree: DraftTree, seed: int, step: int, *,
                out: Optional[TreeResult] = None) -> TreeResult:
    """The lossless walk of each tree with the AR rows p_logits [B, N, V]."""
    if p_logits.dim() != 3:
        raise ValueError("p_logits must be [B, N, V]")
    B, N, V = p_logits.shape
    D = tree.topk_ids.shape[1]
    if N != tree_nodes(D, tree.budget) or tuple(tree.node_token.shape) != (B, N):
        raise ValueError("p_logits must have one row per node slot of the tree")
    dt = _dtype_code(p_logits)
    dev = _check_cuda(p_logits, tree.node_token, tree.node_parent, tree.node_depth,
                      tree.n_nodes)
    for x in (tree.node_token, tree.node_parent, tree.node_depth, tree.n_nodes):
        if x.dtype != torch.int32:
            raise ValueError("tree arrays must be int32")
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = TreeResult(torch.empty((B, D + 1), **i32), torch.empty((B,), **i32),
                         torch.empty((B, N), **i32))
    _check_cuda(out.out_tokens, out.accepted_len, out.node_draw)
    if (tuple(out.out_tokens.shape) != (B, D + 1) or tuple(out.accepted_len.shape) != (B,)
            or tuple(out.node_draw.shape) != (B, N)):
        raise ValueError("out tensors have the wrong shapes")
    st = lib.uno_tree_verify(_ptr(p_logits), _ptr(tree.node_token), _ptr(tree.node_parent),
                             _ptr(tree.node_depth), _ptr(tree.n_nodes), B, D, tree.budget, V, dt,
                             ctypes.c_uint64(seed & (2**64 - 1)),
                             ctypes.c_uint64(step & (2**64 - 1)), _ptr(out.node_draw),
                             _ptr(out.out_tokens), _ptr(out.accepted_len), _stream_handle(dev))
    if st != 0:
        raise UnoError(st, "uno_tree_verify")
    return out


def device_fault_flags(clear: bool = True) -> int:
    """Fault bits set by a kernel wait that gave up (0 = none). Synchronises."""
    flags = ctypes.c_uint(0)
    st = lib.uno_device_fault_flags(1 if clear else 0, ctypes.byref(flags))
    if st != 0:
        raise UnoError(st, "uno_device_fault_flags")
    return int(flags.value)
