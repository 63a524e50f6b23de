"""fp64 CPU oracle for exact attention over contiguous and paged K/V.

TEST INFRASTRUCTURE ONLY. This module is the independent checker of the CUDA
path: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import it.  The library
(``paged_kv_cache_exact_b200``) never imports it and has no CPU fallback.

What it computes is the plain definition of attention, written out in float64
NumPy with the score matrix S and the probability matrix P materialised:

    O = softmax(Q K^T * scale) V

Sources (web pages on the subject; cited by title and section):

* "FlashAttention and PagedAttention: Two Fixes for Two Different Bottlenecks"
  (reactapp.top), section "Why attention is costly": the formula
  softmax(QK^T / sqrt(d)) V.
* "Flash Attention: Fast, Memory-Efficient Attention for LLMs"
  (hiteshsahu.com), section "Standard Attention: The Memory Problem": the three
  steps S = QK^T, P = softmax(S), O = PV; section "The Algorithm": the tiled
  online-softmax recurrence (running max m, running sum l, rescaled output),
  restated here in its unnormalised form (see ``online_softmax_attention_ref``).
* "What is Paged FlashAttention?" (machinoai.in), sections "How does it work?"
  and "Practical example": logical page = token // page_size,
  offset = token % page_size, physical page = block_table[logical page].

Readings adopted where the pages are silent or garbled:

* Causal mask: query row i (0-based, of q_len rows) may see key j (of kv_len
  keys) iff j <= i + (kv_len - q_len).  With q_len == kv_len this is the usual
  lower triangle; with q_len == 1 (decode) every key is visible.
* Physical page layout: ``[num_pages, page_size, H_kv, d]``.  Table padding is
  -1; entries past ceil(seq_len / page_size) are never read.  Tokens of the
  last page at positions >= seq_len are ignored.
* GQA: query head h reads kv head h // (H // H_kv).
* The online-softmax output update printed on the "Flash Attention: Fast,
  Memory-Efficient Attention for LLMs" page, section "The Algorithm", both
  rescales O by l_old / l_new and divides by l again at the end; read literally
  that normalises twice.  The oracle's recurrence keeps O unnormalised
  (O <- e^(m_old - m_new) O + P~ V, final O / l), which is the form the
  page's closing divide and its "reduced non-GEMM FLOPs" remark describe.

Every function here is pinned by tests in ``tests/test_oracle_pins.py``
against values the pages print, closed forms, invariants, brute force and a
library special case (torch CPU float64 SDPA).
"""

from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# Value decoding
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode bfloat16 bit patterns (uint16/int16) to float64, exactly.

    A bfloat16 is the upper 16 bits of an IEEE-754 binary32, so shifting the
    pattern left by 16 gives the float32 with the same value.
    """
    u = np.asarray(bits).view(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def e4m3_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode FP8 e4m3 codes (uint8) to float64, exactly.

    Bit 7 is the sign, bits 6..3 the exponent (bias 7), bits 2..0 the
    mantissa.  Exponent 0 is subnormal (m/8 * 2^-6); exponent 15 with mantissa
    7 is NaN; there are no infinities.
    """
    b = np.asarray(bits).view(np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def to_f64(x: np.ndarray) -> np.ndarray:
    """float arrays are upcast; 16-bit integer arrays are read as bf16 bits."""
    x = np.asarray(x)
    if x.dtype in (np.uint16, np.int16):
        return bf16_bits_to_f64(x)
    return x.astype(np.float64, copy=False)


# ---------------------------------------------------------------------------
# Page-table address resolution
# "What is Paged FlashAttention?", sections "How does it work?" (step 1,
# locate the KV pages) and "Practical example".
# ---------------------------------------------------------------------------

def resolve(block_table_row, page_size: int, token: int) -> tuple[int, int]:
    """Token index -> (physical page, offset inside the page)."""
    logical = token // page_size
    offset = token % page_size
    physical = int(block_table_row[logical])
    return physical, offset


def page_count(seq_len: int, page_size: int) -> tuple[int, int]:
    """Pages a sequence of ``seq_len`` tokens occupies and tokens in its last page.

    "Flash Attention: Fast, Memory-Efficient Attention for LLMs", section
    "PagedAttention (vLLM)": 16-token pages, a 200-token request ends on its
    13th page holding 8 tokens.
    """
    if seq_len <= 0:
        return 0, 0
    n = (seq_len + page_size - 1) // page_size
    return n, seq_len - (n - 1) * page_size


def gather_kv(pages: np.ndarray, block_table_row, seq_len: int, page_size: int) -> np.ndarray:
    """Explicit gather of one sequence's K (or V) rows into a contiguous array.

    ``pages``: ``[num_pages, page_size, H_kv, d]``.  Returns
    ``[H_kv, seq_len, d]`` in float64.  Token t comes from
    ``pages[block_table_row[t // page_size], t % page_size]``.
    This gather is the definition the paged kernels must match without doing it.
    """
    t = np.arange(seq_len)
    table = np.asarray(block_table_row)
    phys = table[t // page_size]
    off = t % page_size
    rows = to_f64(pages[phys, off])            # [seq_len, H_kv, d]
    return np.ascontiguousarray(rows.transpose(1, 0, 2))


# ---------------------------------------------------------------------------
# Dense attention, the plain three-step definition
# "Flash Attention: Fast, Memory-Efficient Attention for LLMs", section
# "Standard Attention: The Memory Problem".
# ---------------------------------------------------------------------------

def allowed_keys(q_len: int, kv_len: int, causal: bool, rows=None) -> np.ndarray:
    """Boolean mask [len(rows), kv_len]: which keys each query row may attend to."""
    i = np.arange(q_len) if rows is None else np.asarray(rows)
    j = np.arange(kv_len)
    if not causal:
        return np.ones((len(i), kv_len), dtype=bool)
    return j[None, :] <= (i[:, None] + (kv_len - q_len))


def softmax_rows(S: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """P = softmax over the allowed entries of each row of S (others get 0)."""
    Sm = np.where(mask, S, NEG_INF)
    mx = Sm.max(axis=1, keepdims=True)
    E = np.where(mask, np.exp(Sm - mx), 0.0)
    return E / E.sum(axis=1, keepdims=True)


def attention_ref(Q, K, V, causal: bool, scale: float, rows=None,
                  row_block: int = 256) -> np.ndarray:
    """One head: Q [q_len, d], K [kv_len, d], V [kv_len, dv] -> O [rows, dv].

    S = Q K^T * scale is formed in row blocks (the whole block of rows against
    all keys), masked, softmaxed and multiplied by V.  ``rows`` selects which
    query rows to compute (all by default).
    """
    Q = to_f64(Q)
    K = to_f64(K)
    V = to_f64(V)
    q_len, kv_len = Q.shape[0], K.shape[0]
    rows = np.arange(q_len) if rows is None else np.asarray(rows)
    out = np.empty((len(rows), V.shape[1]), dtype=np.float64)
    for b0 in range(0, len(rows), row_block):
        r = rows[b0:b0 + row_block]
        S = (Q[r] @ K.T) * scale
        P = softmax_rows(S, allowed_keys(q_len, kv_len, causal, r))
        out[b0:b0 + len(r)] = P @ V
    return out


def mha_ref(Q, K, V, causal: bool, scale: float, rows=None, heads=None) -> np.ndarray:
    """Batched heads: Q [B, H, q_len, d]; K, V [B, H_kv, kv_len, d].

    Returns [B, len(heads), len(rows), d].  Query head h reads kv head
    h // (H // H_kv) (MHA when H_kv == H; "Attention Variants: MHA, GQA, MQA").
    """
    B, H = Q.shape[0], Q.shape[1]
    H_kv = K.shape[1]
    group = H // H_kv
    heads = range(H) if heads is None else heads
    res = []
    for b in range(B):
        res.append(np.stack([attention_ref(Q[b, h], K[b, h // group], V[b, h // group],
                                           causal, scale, rows) for h in heads]))
    return np.stack(res)


# ---------------------------------------------------------------------------
# Paged attention: explicit gather through the block table, then the
# definition.  "What is Paged FlashAttention?", "How does it work?".
# ---------------------------------------------------------------------------

def paged_attention_ref(q, k_pages, v_pages, block_table, seq_lens, page_size: int,
                        causal: bool, scale: float, rows=None, seqs=None,
                        heads=None) -> np.ndarray:
    """q [S, H, q_len, d]; k_pages, v_pages [num_pages, page_size, H_kv, d].

    Sequence s has kv length ``seq_lens[s]`` (the q_len new tokens included)
    and page list ``block_table[s]``.  Returns [len(seqs), len(heads), len(rows), d].
    """
    q = np.asarray(q)
    S, H = q.shape[0], q.shape[1]
    H_kv = k_pages.shape[2]
    group = H // H_kv
    seqs = range(S) if seqs is None else seqs
    heads = range(H) if heads is None else heads
    out = []
    for s in seqs:
        L = int(seq_lens[s])
        Ks = gather_kv(k_pages, block_table[s], L, page_size)
        Vs = gather_kv(v_pages, block_table[s], L, page_size)
        qs = to_f64(q[s])
        out.append(np.stack([attention_ref(qs[h], Ks[h // group], Vs[h // group],
                                           causal, scale, rows) for h in heads]))
    return np.stack(out)


# ---------------------------------------------------------------------------
# The tiled recurrence and the split-K combine (used to pin the algebra the
# kernels follow; not the parity target, which is ``attention_ref``).
# ---------------------------------------------------------------------------

def online_softmax_attention_ref(Q, K, V, causal: bool, scale: float,
                                 tile: int) -> np.ndarray:
    """Tile-by-tile online softmax, in the order of "Flash Attention: Fast,
    Memory-Efficient Attention for LLMs", section "The Algorithm".

    Per key tile j: s = Q K_j^T * scale; m_new = max(m, rowmax s);
    P~ = exp(s - m_new); l = e^(m - m_new) l + rowsum P~;
    O = e^(m - m_new) O + P~ V_j.  Finally O / l.
    Start m = -inf, l = 0, O = 0; the factor e^(m - m_new) is 0 while m = -inf.
    """
    Q, K, V = to_f64(Q), to_f64(K), to_f64(V)
    q_len, kv_len = Q.shape[0], K.shape[0]
    mask_all = allowed_keys(q_len, kv_len, causal)
    m = np.full((q_len, 1), NEG_INF)
    l = np.zeros((q_len, 1))
    O = np.zeros((q_len, V.shape[1]))
    for j0 in range(0, kv_len, tile):
        j1 = min(j0 + tile, kv_len)
        s = np.where(mask_all[:, j0:j1], (Q @ K[j0:j1].T) * scale, NEG_INF)
        m_new = np.maximum(m, s.max(axis=1, keepdims=True))
        alpha = np.where(np.isneginf(m), 0.0, np.exp(np.where(np.isneginf(m), 0.0, m - m_new)))
        safe = np.where(np.isneginf(m_new), 0.0, m_new)
        P = np.where(np.isneginf(s), 0.0, np.exp(s - safe))
        l = alpha * l + P.sum(axis=1, keepdims=True)
        O = alpha * O + P @ V[j0:j1]
        m = m_new
    return O / l


def split_partial_ref(q, K, V, scale: float, lo: int, hi: int):
    """One split of a decode row over keys [lo, hi): (O unnormalised, m, l).

    m = max score over the split, l = sum of e^(s - m), O = sum of e^(s - m) v.
    An empty split returns (0, -inf, 0).
    """
    q, K, V = to_f64(q), to_f64(K), to_f64(V)
    if hi <= lo:
        return np.zeros(V.shape[1]), NEG_INF, 0.0
    s = (K[lo:hi] @ q) * scale
    m = s.max()
    p = np.exp(s - m)
    return p @ V[lo:hi], m, p.sum()


def lse_combine_ref(partials) -> np.ndarray:
    """Merge split partials (O_s, m_s, l_s): m = max m_s,
    l = sum e^(m_s - m) l_s, O = sum e^(m_s - m) O_s / l.  Empty splits
    (m_s = -inf) contribute nothing.  Same algebra as the tile recurrence.
    """
    ms = np.array([p[1] for p in partials], dtype=np.float64)
    m = ms.max()
    w = np.where(np.isneginf(ms), 0.0, np.exp(np.where(np.isneginf(ms), 0.0, ms - m)))
    l = sum(wi * p[2] for wi, p in zip(w, partials))
    O = sum(wi * p[0] for wi, p in zip(w, partials))
    return O / l
