"""The host page allocator (pkv_alloc_*) and its plain model, on the CPU."""

import os
import random

import pytest

import oracle.allocator as OA
from paged_kv_cache_exact_b200 import binding as B

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_allocation.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _requests():
    out = []
    for kind, *rest in _golden():
        if kind == "request":
            ps, tokens, pages, last = rest
            a, b = (int(x) for x in pages.split("-"))
            out.append((int(ps), int(tokens), list(range(a - 1, b)), int(last)))
    return out


@pytest.mark.parametrize("impl", ["model", "library"])
def test_worked_allocation_example(impl):
    reqs = _requests()
    ps = reqs[0][0]
    pool = OA.PagePoolModel(64, ps, 32) if impl == "model" else B.PageAllocator(64, ps, 32)
    for sid, (_, tokens, pages, last) in enumerate(reqs):
        pool.add_seq(sid)
        assert pool.reserve(sid, tokens) == (0, None)
    for sid, (_, tokens, pages, last) in enumerate(reqs):
        if impl == "model":
            row, length = pool.table(sid)
        else:
            rows, lens = pool.block_table([sid])
            row, length = rows[0], lens[0]
        assert row[:len(pages)] == pages and all(x == -1 for x in row[len(pages):])
        assert length == tokens and length - (len(pages) - 1) * ps == last


@pytest.mark.parametrize("impl", ["model", "library"])
def test_shared_prefix_block_tables(impl):
    """Reproduce the printed tables [3, 7, 12] and [3, 7, 9]: with pages 3, 7, 9
    and 12 the smallest free ones, request_2 takes 40 tokens (3 pages, the last
    half full), request_1 forks it and writes one more token: the shared half
    page 9 is copied to 12; blocks 3 and 7 stay shared."""
    shared = {name: [int(x) for x in blocks.split(",")] for kind, name, blocks in
              (r for r in _golden() if r[0] == "shared")}
    pool = OA.PagePoolModel(32, 16, 8) if impl == "model" else B.PageAllocator(32, 16, 8)
    for i in range(13):                         # one page each: ids 0..12
        pool.add_seq(100 + i)
        pool.reserve(100 + i, 1)
    for i in (3, 7, 9, 12):
        pool.free_seq(100 + i)
    pool.add_seq(2)
    assert pool.reserve(2, 40) == (0, None)
    pool.fork(2, 1)
    start, cow = pool.reserve(1, 1)
    assert start == 40 and cow == (9, 12)
    if impl == "model":
        t1, t2 = pool.table(1)[0], pool.table(2)[0]
        refs = pool.refs
    else:
        (t1, t2), _ = pool.block_table([1, 2])
        refs = [pool.page_refs(p) for p in range(32)]
    assert t1[:3] == shared["request_1"] and t2[:3] == shared["request_2"]
    assert refs[3] == refs[7] == 2 and refs[9] == refs[12] == 1


def test_freed_pages_are_reused_smallest_first():
    a = B.PageAllocator(8, 16, 8)
    for s in range(3):
        a.add_seq(s)
        a.reserve(s, 20)                          # 2 pages each: [0,1] [2,3] [4,5]
    a.free_seq(1)
    assert a.num_free() == 4
    a.add_seq(9)
    a.reserve(9, 40)                              # 3 pages: 2, 3, then 6
    assert a.block_table([9])[0][0][:3] == [2, 3, 6]


def test_out_of_pages_changes_nothing():
    a = B.PageAllocator(4, 16, 8)
    a.add_seq(0)
    a.reserve(0, 50)                              # 4 pages
    with pytest.raises(B.PkvError) as e:
        a.reserve(0, 20)
    assert e.value.status == B.PKV_ERR_OUT_OF_PAGES
    assert a.seq_len(0) == 50 and a.num_free() == 0
    with pytest.raises(B.PkvError):
        a.reserve(0, 16 * 8)                      # past max_pages_per_seq
    with pytest.raises(B.PkvError):
        a.add_seq(0)                              # duplicate id


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_the_model(seed):
    rng = random.Random(seed)
    num_pages, ps, max_pages = 48, 16, 12
    lib = B.PageAllocator(num_pages, ps, max_pages)
    mod = OA.PagePoolModel(num_pages, ps, max_pages)
    live, next_id = [], 0
    for _ in range(400):
        op = rng.random()
        if op < 0.15 or not live:
            lib.add_seq(next_id)
            mod.add_seq(next_id)
            live.append(next_id)
            next_id += 1
        elif op < 0.65:
            sid = rng.choice(live)
            n = rng.choice([0, 1, 1, 1, 3, 15, 16, 17, 40])
            try:
                want = mod.reserve(sid, n)
            except (MemoryError, ValueError) as exc:
                with pytest.raises(B.PkvError) as e:
                    lib.reserve(sid, n)
                assert e.value.status == (B.PKV_ERR_OUT_OF_PAGES if isinstance(exc, MemoryError)
                                          else B.PKV_ERR_INVALID_ARG)
                continue
            assert lib.reserve(sid, n) == want
        elif op < 0.8:
            parent = rng.choice(live)
            lib.fork(parent, next_id)
            mod.fork(parent, next_id)
            live.append(next_id)
            next_id += 1
        else:
            sid = live.pop(rng.randrange(len(live)))
            lib.free_seq(sid)
            mod.free_seq(sid)
        assert lib.num_free() == len(mod.free_ids())
        rows, lens = lib.block_table(live)
        for sid, row, length in zip(live, rows, lens):
            assert (row, length) == tuple(mod.table(sid))
        assert [lib.page_refs(p) for p in range(num_pages)] == mod.refs


def test_append_scatter_model_follows_the_worked_mapping():
    """Appending 600 tokens to the [5, 1, 9] table puts token 300 in page 1 at
    offset 44 ("What is Paged FlashAttention?", "Practical example"), and
    reading the sequence back through its table returns the rows in order."""
    import numpy as np
    ps, H, d = 256, 2, 4
    k_pages = np.zeros((10, ps, H, d))
    v_pages = np.zeros((10, ps, H, d))
    rows = np.arange(600 * H * d, dtype=np.float64).reshape(600, H, d)
    kp, vp = OA.append_scatter(k_pages, v_pages, rows, -rows, [0, 600], [0], [[5, 1, 9]], ps)
    assert np.array_equal(kp[1, 44], rows[300]) and np.array_equal(vp[1, 44], -rows[300])
    K, V = OA.logical_kv(kp, vp, [5, 1, 9], 600, ps)
    assert np.array_equal(K, rows) and np.array_equal(V, -rows)
    # appending in two steps (prefill 500, then 100 more) gives the same pools
    kp2, vp2 = OA.append_scatter(k_pages, v_pages, rows[:500], -rows[:500], [0, 500], [0],
                                 [[5, 1, 9]], ps)
    kp2, vp2 = OA.append_scatter(kp2, vp2, rows[500:], -rows[500:], [0, 100], [500],
                                 [[5, 1, 9]], ps)
    assert np.array_equal(kp2, kp) and np.array_equal(vp2, vp)


def test_copy_pages_model():
    import numpy as np
    kp = np.arange(5 * 4 * 2).reshape(5, 4, 2, 1).astype(float)
    k2, v2 = OA.copy_pages(kp, -kp, [1, 3], [4, 0])
    assert np.array_equal(k2[4], kp[1]) and np.array_equal(k2[0], kp[3])
    assert np.array_equal(v2[4], -kp[1]) and np.array_equal(k2[2], kp[2])
