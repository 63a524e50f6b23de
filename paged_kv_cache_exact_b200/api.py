"""Tensor-level convenience over the C ABI (marshalling and output allocation).

Callers that hold torch tensors use these; every step of the computation runs
in ``libpkv.so``.  Outputs (and the decode workspace, unless one is passed)
are allocated with torch on the inputs' device.
"""

from __future__ import annotations

import torch

from . import binding as B

_DT = {torch.bfloat16: B.PKV_BF16, torch.float32: B.PKV_F32}


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _DT[t.dtype]


def prefill(Q, K, V, causal: bool, scale: float, out=None, stream=None) -> torch.Tensor:
    """Contiguous attention, Q/K/V [B, H, N, d] on one CUDA device."""
    Bn, H, N, d = Q.shape
    for t in (Q, K, V):
        assert t.is_contiguous() and t.shape == Q.shape and t.dtype == Q.dtype
    O = torch.empty_like(Q) if out is None else out
    B.attn_prefill(Q, K, V, O, Bn, H, N, d, causal, scale, _dtype(Q), stream)
    return O


def workspace_for(num_seqs: int, H: int, d: int, max_seq_len: int, page_size: int,
                  device) -> torch.Tensor | None:
    n = B.paged_attn_workspace_size(num_seqs, H, d, max_seq_len, page_size)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def paged(q, k_pages, v_pages, block_table, seq_lens, page_size: int, causal: bool,
          scale: float, max_seq_len: int, out=None, workspace=None, stream=None) -> torch.Tensor:
    """Paged attention: q [S, H, q_len, d]; pages [P, page_size, H_kv, d]."""
    S, H, q_len, d = q.shape
    P, ps, H_kv, d2 = k_pages.shape
    assert ps == page_size and d2 == d and v_pages.shape == k_pages.shape
    assert block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32
    assert block_table.is_contiguous() and q.is_contiguous() and k_pages.is_contiguous()
    o = torch.empty_like(q) if out is None else out
    ws = workspace
    if ws is None and q_len == 1:
        ws = workspace_for(S, H, d, max_seq_len, page_size, q.device)
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    B.paged_attn(q, k_pages, v_pages, block_table, seq_lens, page_size, S, q_len, H, H_kv, d,
                 P, block_table.shape[1], max_seq_len, causal, scale, _dtype(q), o, ws,
                 ws_bytes, stream)
    return o
