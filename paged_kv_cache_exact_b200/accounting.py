"""Algorithmic work counts used to turn measured times into roofline fractions.

These count what the method must do, not what a kernel happens to do:

* prefill FLOPs count only the (query, key) pairs the mask allows, at
  2*d multiply-adds for QK^T and 2*d for PV per pair (4*d FLOPs per pair);
* decode bytes count every K and V element of every visible token once, plus
  the query, output, block table and sequence lengths.

The naive three-step traffic model of "FlashAttention vs PagedAttention"
(yourwildcard.ai), section "Count the reads and writes FlashAttention removes"
(8N^2 + 8Nd bytes against 4N^2 d + 3N^2 FLOPs) is kept here too; the tests
check it reproduces the figures that page prints.
"""

from __future__ import annotations


def allowed_pairs(q_len: int, kv_len: int, causal: bool) -> int:
    """Number of (query row, key) pairs attended.  Causal: key j <= i + (kv_len - q_len)."""
    if not causal:
        return q_len * kv_len
    off = kv_len - q_len
    return sum(min(max(i + off + 1, 0), kv_len) for i in range(q_len))


def prefill_flops(B: int, H: int, q_len: int, kv_len: int, d: int, causal: bool) -> int:
    return 4 * d * B * H * allowed_pairs(q_len, kv_len, causal)


def prefill_exps(B: int, H: int, q_len: int, kv_len: int, causal: bool) -> int:
    return B * H * allowed_pairs(q_len, kv_len, causal)


def prefill_min_bytes(B: int, H: int, H_kv: int, q_len: int, kv_len: int, d: int, elem: int = 2) -> int:
    """Compulsory HBM bytes: read Q, K, V once, write O once."""
    return elem * d * (2 * B * H * q_len + 2 * B * H_kv * kv_len)


def decode_bytes(seq_lens, H: int, H_kv: int, d: int, elem: int = 2, max_pages: int = 0) -> int:
    """Bytes a paged decode step must move: all visible K and V rows, q, out,
    the block-table rows and the sequence lengths."""
    total_tokens = sum(int(L) for L in seq_lens)
    S = len(seq_lens)
    kv = 2 * total_tokens * H_kv * d * elem
    qo = 2 * S * H * d * elem
    meta = 4 * S * max_pages + 4 * S
    return kv + qo + meta


def naive_traffic_bytes(N: int, d: int) -> int:
    """Naive three-step attention memory movement (fp16 intermediates): 8N^2 + 8Nd."""
    return 8 * N * N + 8 * N * d


def naive_flops(N: int, d: int) -> int:
    """Naive three-step attention FLOPs: 4 N^2 d + 3 N^2."""
    return 4 * N * N * d + 3 * N * N
