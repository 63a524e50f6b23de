"""The write side of the paged cache on the GPU: appends and page copies are
bit-exact against the oracle's scatter, and a cache built step by step with the
allocator (prefill chunk, decode steps, a forked sequence with copy-on-write)
gives the same decode attention as the oracle on the logical sequences."""

import numpy as np
import pytest
import torch

import oracle
import oracle.allocator as OA
from paged_kv_cache_exact_b200 import api
from tests._util import check_close, np_of

pytestmark = pytest.mark.gpu

DT = {torch.bfloat16: 1, torch.float32: 0}


def _append(kp, vp, k_new, v_new, cu, start, table, ps):
    from paged_kv_cache_exact_b200 import binding as B
    dev = kp.device
    cu_t = torch.tensor(cu, dtype=torch.int32, device=dev)
    st_t = torch.tensor(start, dtype=torch.int32, device=dev)
    tb_t = torch.tensor(table, dtype=torch.int32, device=dev)
    B.paged_kv_append(k_new, v_new, cu_t, st_t, tb_t, tb_t.shape[1], len(start), k_new.shape[0],
                      kp, vp, kp.shape[0], ps, kp.shape[2], kp.shape[3], DT[kp.dtype])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("ps", [16, 256])
def test_append_bit_exact(dtype, ps):
    from paged_kv_cache_exact_b200 import binding as B
    g = torch.Generator().manual_seed(91)
    P, H_kv, d = 40, 4, 128 if dtype == torch.bfloat16 else 64
    kp = torch.randn(P, ps, H_kv, d, generator=g).to(dtype)
    vp = torch.randn(P, ps, H_kv, d, generator=g).to(dtype)
    # three sequences: prefill 37 tokens, decode 1 token at a page edge, 300 tokens mid-page
    counts, start = [37, 1, 300], [0, 2 * ps - 1, 5]
    # distinct shuffled pages, enough to cover each sequence's last new position
    perm = torch.randperm(P, generator=g).tolist()
    need = [(st + n - 1) // ps + 1 for st, n in zip(start, counts)]
    width = max(need)
    tables, cur = [], 0
    for n_pages in need:
        tables.append(perm[cur:cur + n_pages] + [-1] * (width - n_pages))
        cur += n_pages
    cu = [0, 37, 38, 338]
    k_new = torch.randn(338, H_kv, d, generator=g).to(dtype)
    v_new = torch.randn(338, H_kv, d, generator=g).to(dtype)
    want_k, want_v = OA.append_scatter(np_of(kp), np_of(vp), np_of(k_new), np_of(v_new), cu,
                                       start, tables, ps)
    kd, vd = kp.cuda(), vp.cuda()
    _append(kd, vd, k_new.cuda(), v_new.cuda(), cu, start, tables, ps)
    torch.cuda.synchronize()
    assert np.array_equal(np_of(kd), want_k) and np.array_equal(np_of(vd), want_v)
    assert B.pkv_last_device_error()[0] == 0


def test_append_bad_page_is_skipped_and_flagged():
    from paged_kv_cache_exact_b200 import binding as B
    kp = torch.zeros(4, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    k_new = torch.ones(2, 2, 128, dtype=torch.bfloat16, device="cuda")
    B.pkv_last_device_error()
    _append(kp, vp, k_new, k_new, [0, 1, 2], [0, 0], [[1], [99]], 16)
    st, bits = B.pkv_last_device_error()
    assert st == B.PKV_ERR_BAD_TABLE and bits & B.PKV_DEVERR_BAD_PAGE
    assert kp[1, 0].float().eq(1).all() and kp.float().sum() == 2 * 128


def test_copy_pages_bit_exact():
    from paged_kv_cache_exact_b200 import binding as B
    g = torch.Generator().manual_seed(92)
    kp = torch.randn(12, 16, 8, 128, generator=g).to(torch.bfloat16)
    vp = torch.randn(12, 16, 8, 128, generator=g).to(torch.bfloat16)
    src, dst = [1, 5, 7], [9, 0, 11]
    want_k, want_v = OA.copy_pages(np_of(kp), np_of(vp), src, dst)
    kd, vd = kp.cuda(), vp.cuda()
    B.paged_kv_copy_pages(kd, vd, torch.tensor(src, dtype=torch.int32, device="cuda"),
                          torch.tensor(dst, dtype=torch.int32, device="cuda"), 3, 12, 16, 8,
                          128, 1)
    torch.cuda.synchronize()
    assert np.array_equal(np_of(kd), want_k) and np.array_equal(np_of(vd), want_v)


def test_serving_simulation_with_fork_and_copy_on_write():
    """Allocator + append + copy + decode: two prompts are prefilled in chunks,
    a third sequence forks the first mid-page, then all decode 20 steps; every
    step's decode output matches the oracle on the logical K/V."""
    from paged_kv_cache_exact_b200 import binding as B
    ps, H, H_kv, d, P, max_pages = 16, 8, 4, 128, 96, 32
    g = torch.Generator().manual_seed(93)
    alloc = B.PageAllocator(P, ps, max_pages)
    kp = torch.full((P, ps, H_kv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vp = torch.full_like(kp, float("nan"))
    logical = {}                                   # seq -> list of (k_row, v_row) on the CPU

    def write(sid_rows):
        """sid_rows: {sid: (k [n,H_kv,d], v)} -> reserve, copy-on-write, append."""
        sids = list(sid_rows)
        starts, cu, ks, vs, cows = [], [0], [], [], []
        for sid in sids:
            k, v = sid_rows[sid]
            start, cow = alloc.reserve(sid, k.shape[0])
            if cow:
                cows.append(cow)
            starts.append(start)
            cu.append(cu[-1] + k.shape[0])
            ks.append(k)
            vs.append(v)
            logical.setdefault(sid, []).extend(zip(k, v))
        if cows:
            B.paged_kv_copy_pages(kp, vp, torch.tensor([c[0] for c in cows], dtype=torch.int32, device="cuda"),
                                  torch.tensor([c[1] for c in cows], dtype=torch.int32, device="cuda"),
                                  len(cows), P, ps, H_kv, d, 1)
        rows, _ = alloc.block_table(sids)
        _append(kp, vp, torch.cat(ks).cuda(), torch.cat(vs).cuda(), cu, starts, rows, ps)

    def rand(n):
        return (torch.randn(n, H_kv, d, generator=g).to(torch.bfloat16),
                torch.randn(n, H_kv, d, generator=g).to(torch.bfloat16))

    alloc.add_seq(0)
    alloc.add_seq(1)
    write({0: rand(100), 1: rand(37)})            # prefill chunk 1
    write({0: rand(21)})                          # prefill chunk 2: 121 tokens, mid-page
    alloc.fork(0, 2)                              # shares 8 pages incl. the half-full last one
    logical[2] = list(logical[0])
    for step in range(20):
        write({0: rand(1), 1: rand(1), 2: rand(1)})   # step 0 copies the shared half page
        sids = [0, 1, 2]
        rows, lens = alloc.block_table(sids)
        q = torch.randn(3, H, 1, d, generator=g).to(torch.bfloat16)
        out = api.paged(q.cuda(), kp, vp, torch.tensor(rows, dtype=torch.int32, device="cuda"),
                        torch.tensor(lens, dtype=torch.int32, device="cuda"), ps, True,
                        d ** -0.5, max_seq_len=max(lens)).cpu()
        want = np.zeros((3, H, 1, d))
        for i, sid in enumerate(sids):
            K = np.stack([oracle.to_f64(np_of(k)) for k, _ in logical[sid]])
            V = np.stack([oracle.to_f64(np_of(v)) for _, v in logical[sid]])
            assert K.shape[0] == lens[i]
            for h in range(H):
                want[i, h] = oracle.attention_ref(np_of(q[i, h]), K[:, h // 2], V[:, h // 2],
                                                  True, d ** -0.5)
        check_close(out, want, f"decode step {step}")
    assert alloc.page_refs(rows[0][0]) == 2           # prefix still shared by seqs 0 and 2
    assert B.pkv_last_device_error()[0] == 0
