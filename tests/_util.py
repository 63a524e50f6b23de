"""Helpers shared by the GPU parity tests."""

import numpy as np
import torch

import oracle

# Tolerances (elementwise, |got - want| <= ATOL + RTOL * |want|):
# bf16 inputs with float32 accumulation and a bf16 output: 1e-2 + 2e-2 |o|;
# the float32 path: 2e-3 absolute.
BF16_ATOL, BF16_RTOL = 1e-2, 2e-2
F32_ATOL = 2e-3


def np_of(t: torch.Tensor) -> np.ndarray:
    """CPU numpy view the oracle reads: bf16 as raw bits, float32 as is."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    return t.numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return oracle.to_f64(np_of(t))


def check_close(got: torch.Tensor, want: np.ndarray, what: str = ""):
    g = f64(got)
    assert g.shape == want.shape, (g.shape, want.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - want)
    if got.dtype == torch.bfloat16:
        bound = BF16_ATOL + BF16_RTOL * np.abs(want)
    else:
        bound = np.full_like(want, F32_ATOL)
    bad = err > bound
    big = np.abs(want) >= 0.5
    rel = float((err[big] / np.abs(want[big])).max()) if big.any() else 0.0
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements out of tolerance; "
                           f"max abs err {err.max():.3e}, max rel err (|o|>=0.5) {rel:.3e}")
    return float(err.max()), rel


def paged_ref_per_head(w, seqs=None, heads=None, rows=None):
    """Oracle for a PagedInputs, one head at a time (bounded host memory).

    Returns [len(seqs), len(heads), rows, d] float64.
    """
    S, H = w.q.shape[0], w.q.shape[1]
    H_kv = w.k_pages.shape[2]
    group = H // H_kv
    seqs = list(range(S)) if seqs is None else list(seqs)
    heads = list(range(H)) if heads is None else list(heads)
    kp, vp, q = np_of(w.k_pages), np_of(w.v_pages), np_of(w.q)
    table, lens = w.block_table.numpy(), w.seq_lens.numpy()
    out = np.empty((len(seqs), len(heads), w.q.shape[2] if rows is None else len(rows),
                    w.q.shape[3]))
    for hi, h in enumerate(heads):
        kvh = h // group
        r = oracle.paged_attention_ref(q[:, h:h + 1], kp[:, :, kvh:kvh + 1], vp[:, :, kvh:kvh + 1],
                                       table, lens, w.page_size, w.causal, w.scale,
                                       rows=rows, seqs=seqs)
        out[:, hi] = r[:, 0]
    return out


def to_dev(w, device="cuda"):
    """Move a PagedInputs' tensors to the GPU (returns a dict)."""
    return dict(q=w.q.to(device), k=w.k_pages.to(device), v=w.v_pages.to(device),
                table=w.block_table.to(device), lens=w.seq_lens.to(device))
