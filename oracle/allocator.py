"""Plain model of the paged KV cache's bookkeeping (test infrastructure only).

Written from "FlashAttention and PagedAttention: Two Fixes for Two Different
Bottlenecks", section "PagedAttention ... How it works" (fixed-size blocks, a
per-sequence block table, allocation on demand, shared prefixes copied only
when they diverge) and "Flash Attention: Fast, Memory-Efficient Attention for
LLMs", section "PagedAttention (vLLM)" (pages of finished sequences are freed
and reused; a 200-token request on 16-token pages ends on a 13th page holding
8 tokens).

Readings where the pages are silent: the next page handed out is the
smallest free id; pages carry reference counts; a sequence about to write
into a shared, partially filled last page first gets a private copy of it.

Also here: the device-side effect of appending tokens, written as the plain
scatter it is (token at position pos of sequence s lands in page
block_table[s][pos // page_size] at offset pos % page_size).
"""

from __future__ import annotations

import numpy as np


class PagePoolModel:
    def __init__(self, num_pages: int, page_size: int, max_pages: int):
        self.page_size = page_size
        self.max_pages = max_pages
        self.refs = [0] * num_pages
        self.seqs: dict[int, list] = {}     # id -> [pages, length]

    def free_ids(self):
        return [p for p, r in enumerate(self.refs) if r == 0]

    def add_seq(self, sid):
        if sid in self.seqs:
            raise KeyError(sid)
        self.seqs[sid] = [[], 0]

    def reserve(self, sid, n):
        """Grow a sequence by n tokens; returns (start_pos, (src, dst) or None)."""
        pages, length = self.seqs[sid]
        new_len = length + n
        need = -(-new_len // self.page_size)
        if need > self.max_pages:
            raise ValueError("table too short")
        shared_tail = n > 0 and length % self.page_size != 0 and self.refs[pages[-1]] > 1
        extra = need - len(pages) + (1 if shared_tail else 0)
        free = self.free_ids()
        if extra > len(free):
            raise MemoryError("out of pages")
        cow = None
        if shared_tail:
            fresh = free.pop(0)
            self.refs[fresh] = 1
            self.refs[pages[-1]] -= 1
            cow = (pages[-1], fresh)
            pages[-1] = fresh
        while len(pages) < need:
            p = free.pop(0)
            self.refs[p] = 1
            pages.append(p)
        self.seqs[sid][1] = new_len
        return length, cow

    def fork(self, parent, child):
        if child in self.seqs:
            raise KeyError(child)
        pages, length = self.seqs[parent]
        for p in pages:
            self.refs[p] += 1
        self.seqs[child] = [list(pages), length]

    def free_seq(self, sid):
        pages, _ = self.seqs.pop(sid)
        for p in pages:
            self.refs[p] -= 1

    def table(self, sid):
        pages, length = self.seqs[sid]
        return pages + [-1] * (self.max_pages - len(pages)), length


def append_scatter(k_pages, v_pages, k_new, v_new, cu_new, start_pos, block_table, page_size):
    """Expected pools after appending: row r of sequence s goes to position
    start_pos[s] + (r - cu_new[s]).  Returns new (k_pages, v_pages) arrays."""
    kp, vp = k_pages.copy(), v_pages.copy()
    for s in range(len(cu_new) - 1):
        for r in range(cu_new[s], cu_new[s + 1]):
            pos = start_pos[s] + (r - cu_new[s])
            phys = block_table[s][pos // page_size]
            kp[phys, pos % page_size] = k_new[r]
            vp[phys, pos % page_size] = v_new[r]
    return kp, vp


def copy_pages(k_pages, v_pages, src, dst):
    kp, vp = k_pages.copy(), v_pages.copy()
    for a, b in zip(src, dst):
        kp[b] = k_pages[a]
        vp[b] = v_pages[a]
    return kp, vp


def logical_kv(k_pages, v_pages, block_table_row, seq_len, page_size):
    """A sequence's K/V as [seq_len, H_kv, d] through its table (for checks)."""
    t = np.arange(seq_len)
    phys = np.asarray(block_table_row)[t // page_size]
    return k_pages[phys, t % page_size], v_pages[phys, t % page_size]
