"""Seeded synthetic inputs for the attention paths (no attention arithmetic here).

Both the CUDA path (through the tests and ``bench.py``) and the fp64 oracle are
fed from these generators; nothing in this module computes attention.

Every tensor is drawn on the CPU from ``torch.Generator().manual_seed(seed)``
in a fixed order, values ~ N(0, 1) in float32, then rounded to bfloat16 (RNE)
where the workload is bf16.  Paged workloads lay K/V out as
``[num_pages, page_size, H_kv, d]``; the block table is int32
``[num_seqs, max_pages]`` padded with -1.  Pool pages no sequence uses, and the
tail of each sequence's last page past ``seq_len``, are filled with NaN
("poison"): any read the table does not allow shows up as NaN in the output.

The five named workloads follow the configurations the attention pages are
measured on (shapes, page sizes, length mixes).  Draw order:

* dense:  Q, K, V.
* paged:  seq_lens, pool permutation, q, K pool, V pool (K/V pools drawn in
  chunks of 64 pages so large pools need no float32 copy of the whole pool).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

POISON = float("nan")


@dataclass
class DenseInputs:
    """Contiguous [B, H, N, d] Q/K/V (K/V may have H_kv heads)."""
    Q: torch.Tensor
    K: torch.Tensor
    V: torch.Tensor
    causal: bool
    scale: float

    @property
    def shape(self):
        B, H, N, d = self.Q.shape
        return B, H, N, d


@dataclass
class PagedInputs:
    """Paged K/V cache plus per-sequence block tables."""
    q: torch.Tensor               # [S, H, q_len, d]
    k_pages: torch.Tensor         # [num_pages, page_size, H_kv, d]
    v_pages: torch.Tensor
    block_table: torch.Tensor     # int32 [S, max_pages], -1 padded
    seq_lens: torch.Tensor        # int32 [S]
    page_size: int
    causal: bool
    scale: float
    decoy_pages: list = field(default_factory=list)

    @property
    def num_seqs(self):
        return self.q.shape[0]

    @property
    def q_len(self):
        return self.q.shape[2]

    @property
    def max_seq_len(self):
        return int(self.seq_lens.max())


def _randn(gen, shape, dtype):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    return x.to(dtype)


def make_dense(seed: int, B: int, H: int, N: int, d: int, dtype=torch.bfloat16,
               causal: bool = True, scale: float | None = None, H_kv: int | None = None,
               N_kv: int | None = None) -> DenseInputs:
    gen = torch.Generator().manual_seed(seed)
    H_kv = H if H_kv is None else H_kv
    N_kv = N if N_kv is None else N_kv
    Q = _randn(gen, (B, H, N, d), dtype)
    K = _randn(gen, (B, H_kv, N_kv, d), dtype)
    V = _randn(gen, (B, H_kv, N_kv, d), dtype)
    return DenseInputs(Q, K, V, causal, d ** -0.5 if scale is None else scale)


def _fill_pool(gen, pool, dtype, chunk=64):
    num_pages = pool.shape[0]
    for p0 in range(0, num_pages, chunk):
        p1 = min(num_pages, p0 + chunk)
        pool[p0:p1] = _randn(gen, (p1 - p0,) + tuple(pool.shape[1:]), dtype)


def make_paged(seed: int, seq_lens, H: int, d: int, page_size: int, q_len: int = 1,
               dtype=torch.bfloat16, H_kv: int | None = None, causal: bool = True,
               scale: float | None = None, decoys: int = 8, poison: bool = True,
               fixed_tables: dict | None = None, pool_pages: int | None = None) -> PagedInputs:
    """Paged workload.

    ``seq_lens``: list of ints, or a (lo, hi, count) tuple drawn uniformly
    from [lo, hi] with the generator.  ``fixed_tables`` maps a sequence index to
    an explicit page list (e.g. {0: [5, 1, 9]}); those pages are excluded from
    the shuffled pool the other sequences draw from.  ``pool_pages`` forces the
    pool size (default: exactly the pages needed plus ``decoys``).
    """
    gen = torch.Generator().manual_seed(seed)
    H_kv = H if H_kv is None else H_kv
    fixed_tables = fixed_tables or {}
    if isinstance(seq_lens, tuple):
        lo, hi, count = seq_lens
        lens = torch.randint(lo, hi + 1, (count,), generator=gen, dtype=torch.int64).tolist()
    else:
        lens = [int(x) for x in seq_lens]
    S = len(lens)
    need = [(L + page_size - 1) // page_size for L in lens]
    for s, pages in fixed_tables.items():
        assert len(pages) >= need[s], "fixed table shorter than its sequence"
    fixed_ids = sorted({p for pages in fixed_tables.values() for p in pages})
    free_needed = sum(n for s, n in enumerate(need) if s not in fixed_tables)
    num_pages = free_needed + len(fixed_ids) + decoys
    if fixed_ids:
        num_pages = max(num_pages, max(fixed_ids) + 1 + decoys)
    if pool_pages is not None:
        assert pool_pages >= num_pages - decoys
        num_pages = pool_pages
    perm = torch.randperm(num_pages, generator=gen).tolist()
    fixed_set = set(fixed_ids)
    free = [p for p in perm if p not in fixed_set]
    max_pages = max(need) if need else 1
    table = torch.full((S, max(max_pages, 1)), -1, dtype=torch.int32)
    cursor = 0
    for s in range(S):
        if s in fixed_tables:
            pages = list(fixed_tables[s])[:need[s]]
        else:
            pages = free[cursor:cursor + need[s]]
            cursor += need[s]
        table[s, :len(pages)] = torch.tensor(pages, dtype=torch.int32)
    used = set(table[table >= 0].tolist())
    decoy_pages = [p for p in range(num_pages) if p not in used]

    q = _randn(gen, (S, H, q_len, d), dtype)
    k_pages = torch.empty((num_pages, page_size, H_kv, d), dtype=dtype)
    v_pages = torch.empty((num_pages, page_size, H_kv, d), dtype=dtype)
    _fill_pool(gen, k_pages, dtype)
    _fill_pool(gen, v_pages, dtype)
    if poison:
        for p in decoy_pages:
            k_pages[p] = POISON
            v_pages[p] = POISON
        for s in range(S):
            if lens[s] % page_size:
                last = int(table[s, need[s] - 1])
                k_pages[last, lens[s] % page_size:] = POISON
                v_pages[last, lens[s] % page_size:] = POISON
    return PagedInputs(q, k_pages, v_pages, table,
                       torch.tensor(lens, dtype=torch.int32), page_size, causal,
                       d ** -0.5 if scale is None else scale, decoy_pages)


# ---------------------------------------------------------------------------
# The five named workloads.
# ---------------------------------------------------------------------------

WORKLOADS = {
    1: "tiny exact check: 1x1x256x64 fp32, non-causal; paged ps=16 over a permuted 16-page pool",
    2: "causal prefill: B=4 H=32 N=4096 d=128 bf16, contiguous [B,H,N,d]",
    3: "paged decode: 64 seqs x 32 heads, d=128 bf16, seq_lens U[512,8192], page_size=16",
    4: "paged decode, large pages: 16 seqs x 32 heads, d=128 bf16, seq_lens U[600,32768], "
       "page_size=256, seq 0 = 600 tokens on pages [5,1,9]",
    5: "long-context paged causal prefill: 1x32x32768x128 bf16, 128 pages of 256 "
       "(shuffled, from a 256-page pool)",
}


def workload(i: int):
    """Inputs of named workload ``i`` (seed 1000 + i)."""
    seed = 1000 + i
    if i == 1:
        dense = make_dense(seed, 1, 1, 256, 64, dtype=torch.float32, causal=False, scale=0.125)
        # Paged copy of the same K/V: 16 pages of 16 tokens, table = a permutation.
        gen = torch.Generator().manual_seed(seed + 100)
        table = torch.randperm(16, generator=gen).to(torch.int32)
        k_pages = torch.empty((16, 16, 1, 64), dtype=torch.float32)
        v_pages = torch.empty((16, 16, 1, 64), dtype=torch.float32)
        for lp in range(16):
            k_pages[int(table[lp]), :, 0] = dense.K[0, 0, lp * 16:(lp + 1) * 16]
            v_pages[int(table[lp]), :, 0] = dense.V[0, 0, lp * 16:(lp + 1) * 16]
        paged = PagedInputs(dense.Q.clone(), k_pages, v_pages, table[None, :].clone(),
                            torch.tensor([256], dtype=torch.int32), 16, False, 0.125, [])
        return dense, paged
    if i == 2:
        return make_dense(seed, 4, 32, 4096, 128, causal=True)
    if i == 3:
        return make_paged(seed, (512, 8192, 64), 32, 128, 16, q_len=1, decoys=64)
    if i == 4:
        return make_paged(seed, [600] + list(_draw_lens(seed, 600, 32768, 15)), 32, 128, 256,
                          q_len=1, decoys=8, fixed_tables={0: [5, 1, 9]})
    if i == 5:
        return make_paged(seed, [32768], 32, 128, 256, q_len=32768, decoys=128,
                          pool_pages=256)
    raise KeyError(i)


def _draw_lens(seed, lo, hi, count):
    gen = torch.Generator().manual_seed(seed + 7)
    return torch.randint(lo, hi + 1, (count,), generator=gen, dtype=torch.int64).tolist()
