"""Paged decode (q_len = 1, bf16) on the GPU against the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_exact_b200.workloads import make_paged, workload
from tests._util import check_close, np_of, paged_ref_per_head, to_dev

pytestmark = pytest.mark.gpu


def _run(w, **kw):
    from paged_kv_cache_exact_b200 import api
    d = to_dev(w)
    out = api.paged(d["q"], d["k"], d["v"], d["table"], d["lens"], w.page_size, w.causal,
                    w.scale, max_seq_len=kw.get("max_seq_len", w.max_seq_len))
    torch.cuda.synchronize()
    return out.cpu()


def _device_status():
    from paged_kv_cache_exact_b200 import binding as B
    return B.pkv_last_device_error()


@pytest.mark.parametrize("ps", [16, 64, 256])
@pytest.mark.parametrize("lens", [[1, 15, 16, 17], [300, 1000, 31, 4097], [2049]])
def test_decode_small(ps, lens):
    w = make_paged(11, lens, H=4, d=128, page_size=ps, q_len=1, decoys=3)
    got = _run(w)
    check_close(got, paged_ref_per_head(w), f"decode ps={ps} lens={lens}")
    assert _device_status()[0] == 0


def test_decode_gqa():
    w = make_paged(12, [777, 64, 5000], H=32, H_kv=8, d=128, page_size=16, q_len=1)
    check_close(_run(w), paged_ref_per_head(w), "decode gqa 32/8")


def test_decode_aliased_pages():
    """Two sequences share physical pages for a common prefix (pages 3 and 7,
    as in the block-table example of "FlashAttention and PagedAttention: Two
    Fixes for Two Different Bottlenecks"); pages are read-only, results exact."""
    w = make_paged(13, [48, 48], H=2, d=128, page_size=16, q_len=1, decoys=0,
                   fixed_tables={0: [3, 7, 12], 1: [3, 7, 9]}, pool_pages=13)
    check_close(_run(w), paged_ref_per_head(w), "decode aliased")


def test_decode_many_splits_and_max_len_slack():
    # max_seq_len larger than any actual length: extra splits must be empty
    w = make_paged(14, [5, 9000, 100], H=2, d=128, page_size=32, q_len=1)
    pad = torch.full((3, 512 - w.block_table.shape[1]), -1, dtype=torch.int32)
    w.block_table = torch.cat([w.block_table, pad], dim=1).contiguous()
    check_close(_run(w, max_seq_len=16384), paged_ref_per_head(w), "decode slack")


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [3, 4])
def test_decode_full_workloads(cfg):
    w = workload(cfg)
    got = _run(w)
    err, rel = check_close(got, paged_ref_per_head(w), f"workload {cfg}")
    assert _device_status()[0] == 0
    print(f"workload {cfg}: max abs err {err:.3e}, max rel err {rel:.3e}")


def _sentinel_case(ps, lens, H, seed):
    """Pages where each (seq, head) has one key that dominates by > 200 in the
    exponent; its V row encodes (physical page, offset, seq, head) as small
    integers exact in bf16, so the output must equal that row bit for bit."""
    w = make_paged(seed, lens, H=H, d=128, page_size=ps, q_len=1, decoys=2)
    table = w.block_table.numpy()
    w.q[:] = 1.0
    w.scale = 1.0
    used = sorted(set(table[table >= 0].tolist()))
    for p in used:                     # clear used pages (tails stay poisoned)
        w.k_pages[p] = torch.where(torch.isnan(w.k_pages[p].float()), w.k_pages[p],
                                   torch.zeros_like(w.k_pages[p]))
        w.v_pages[p] = torch.where(torch.isnan(w.v_pages[p].float()), w.v_pages[p],
                                   torch.zeros_like(w.v_pages[p]))
    expect = np.zeros((len(lens), H, 1, 128))
    rng = np.random.default_rng(seed)
    for s, L in enumerate(lens):
        for h in range(H):
            # sweep page boundaries: first/last token of a page, and random ones
            cands = [0, L - 1, min(L - 1, ps - 1), min(L - 1, ps), int(rng.integers(L))]
            t = cands[(s * H + h) % len(cands)]
            phys, off = oracle.resolve(table[s], ps, t)
            w.k_pages[phys, off, h] = 2.0          # score 256 vs 0 elsewhere
            code = [phys % 16, (phys // 16) % 16, (phys // 256) % 16, phys // 4096,
                    off, s, h]
            w.v_pages[phys, off, h, :7] = torch.tensor(code, dtype=torch.float32).to(w.v_pages.dtype)
            expect[s, h, 0, :7] = code
    return w, expect


@pytest.mark.parametrize("ps,lens", [(256, [600, 300, 1]), (16, [33, 1024, 17, 999])])
def test_sentinel_address_probe_bit_exact(ps, lens):
    w, expect = _sentinel_case(ps, lens, H=4, seed=15)
    got = _run(w).double().numpy()
    assert np.array_equal(got, expect)


def test_sentinel_worked_example_token_300():
    """Token 300 of the 600-token sequence on pages [5, 1, 9] is read from
    physical page 1, offset 44 (printed example), through the kernel."""
    w = make_paged(16, [600], H=1, d=128, page_size=256, q_len=1, decoys=2,
                   fixed_tables={0: [5, 1, 9]})
    w.q[:] = 1.0
    w.scale = 1.0
    for p in (5, 1, 9):
        w.k_pages[p] = torch.where(torch.isnan(w.k_pages[p].float()), w.k_pages[p],
                                   torch.zeros_like(w.k_pages[p]))
        w.v_pages[p] = torch.where(torch.isnan(w.v_pages[p].float()), w.v_pages[p],
                                   torch.zeros_like(w.v_pages[p]))
    w.k_pages[1, 44, 0] = 2.0
    w.v_pages[1, 44, 0, 0] = 1.0      # physical page
    w.v_pages[1, 44, 0, 1] = 44.0     # offset
    got = _run(w)[0, 0, 0, :2].double().tolist()
    assert got == [1.0, 44.0]


def test_bad_page_id_is_flagged_not_faulted():
    from paged_kv_cache_exact_b200 import binding as B
    w = make_paged(17, [64, 64], H=2, d=128, page_size=16, q_len=1)
    w.block_table[1, 2] = w.k_pages.shape[0] + 5          # out of range for seq 1
    _device_status()                                       # clear
    got = _run(w)
    st, bits = _device_status()
    assert st == B.PKV_ERR_BAD_TABLE and bits & B.PKV_DEVERR_BAD_PAGE
    # sequence 0 is untouched by the bad entry
    check_close(got[:1], paged_ref_per_head(w, seqs=[0]), "good sequence")


@pytest.mark.parametrize("ps,bad_page", [(16, 0), (16, 5), (256, 1)])
def test_grouped_decode_bad_page_is_left_out_and_flagged(ps, bad_page):
    """Grouped heads (8 query heads over 2 kv heads) with a page id outside the
    pool in sequence 1's table: flagged, sequence 0 untouched, and sequence 1
    is attention over its other tokens (decode sees every token, so leaving
    the page's tokens out equals the oracle on the shortened sequence).  Page
    0 is every split's first page of that sequence, so a warp starts on it."""
    from paged_kv_cache_exact_b200 import binding as B
    w = make_paged(18 + ps, [700, 1500], H=8, H_kv=2, d=128, page_size=ps, q_len=1)
    _device_status()                                       # clear
    w.block_table[1, bad_page] = w.k_pages.shape[0] + 3
    got = _run(w)
    st, bits = _device_status()
    assert st == B.PKV_ERR_BAD_TABLE and bits & B.PKV_DEVERR_BAD_PAGE
    check_close(got[:1], paged_ref_per_head(w, seqs=[0]), "good sequence")
    L = int(w.seq_lens[1])
    drop = set(range(bad_page * ps, (bad_page + 1) * ps))
    keep = np.array([t for t in range(L) if t not in drop])
    table = w.block_table[1].numpy().copy()
    table[table >= w.k_pages.shape[0]] = 0                 # any page: its tokens are dropped
    K = oracle.gather_kv(np_of(w.k_pages), table, L, ps)[:, keep]
    V = oracle.gather_kv(np_of(w.v_pages), table, L, ps)[:, keep]
    q = oracle.to_f64(np_of(w.q[1]))
    want = np.stack([oracle.attention_ref(q[h], K[h // 4], V[h // 4], True, w.scale)
                     for h in range(8)])
    check_close(got[1], want, "sequence with a bad page")


@pytest.mark.parametrize("H,H_kv", [(8, 4), (16, 4), (32, 4), (16, 1), (64, 2)])
@pytest.mark.parametrize("ps", [16, 256])
def test_decode_grouped_heads(H, H_kv, ps):
    """Query heads sharing a kv head (2, 4, 8, 16 and 32 per kv head; the last
    spans two CTAs of 16), ragged lengths including 1 and page edges."""
    w = make_paged(18 + H, [1, 17, 300, 4097, 2 * ps], H=H, H_kv=H_kv, d=128, page_size=ps,
                   q_len=1, decoys=3)
    check_close(_run(w), paged_ref_per_head(w), f"decode H={H} H_kv={H_kv} ps={ps}")
    assert _device_status()[0] == 0


def test_decode_grouped_long_split_boundaries():
    """Grouped heads with enough (sequence, kv head) pairs that the CTAs take
    2048-key splits (eight times the per-head plan's 256): lengths on every edge of
    that plan (one key, a multiple of 2048, one past it, one short of it) and
    random ones, merged by the combine."""
    edge = [1, 511, 512, 513, 2047, 2048, 2049, 2560, 4096, 4097, 6143, 9000]
    lens = edge + torch.randint(1, 9001, (64 - len(edge),),
                                generator=torch.Generator().manual_seed(5)).tolist()
    w = make_paged(31, lens, H=16, H_kv=4, d=128, page_size=16, q_len=1, decoys=8)
    check_close(_run(w), paged_ref_per_head(w), "decode grouped, 2048-key splits")
    assert _device_status()[0] == 0


@pytest.mark.slow
def test_decode_grouped_full_size():
    """64 sequences x 64 query heads over 8 kv heads (Llama-3-70B-like), lengths
    U[512, 8192], pages of 16."""
    w = make_paged(2003, (512, 8192, 64), 64, 128, 16, q_len=1, H_kv=8, decoys=64)
    err, rel = check_close(_run(w), paged_ref_per_head(w), "decode gqa 64/8 full size")
    assert _device_status()[0] == 0
    print(f"gqa 64/8: max abs err {err:.3e}, max rel err {rel:.3e}")


@pytest.mark.parametrize("H,H_kv", [(8, 8), (16, 2)])
def test_decode_captured_in_a_cuda_graph_matches_direct_calls(H, H_kv):
    """Decode captured into a CUDA graph and replayed gives the direct call's
    bits: per-head heads (split kernel, then a plain merge launch) and grouped
    heads (split kernel, then the merge as a programmatic dependent launch),
    with several splits per sequence so that the merge runs."""
    from paged_kv_cache_exact_b200 import api
    w = make_paged(41 + H, [700, 3000, 5000, 1], H=H, H_kv=H_kv, d=128, page_size=16, q_len=1,
                   decoys=4)
    d = to_dev(w)
    ws = api.workspace_for(w.num_seqs, H, 128, w.max_seq_len, 16, d["q"].device)
    assert ws is not None                                      # several splits per sequence
    out = torch.empty_like(d["q"])

    def call():
        api.paged(d["q"], d["k"], d["v"], d["table"], d["lens"], 16, True, w.scale,
                  max_seq_len=w.max_seq_len, out=out, workspace=ws)

    call()                                                     # first call outside the capture
    torch.cuda.synchronize()
    direct = out.clone()
    out.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), direct.view(torch.int16))
    check_close(out.cpu(), paged_ref_per_head(w), f"graph-replayed decode H={H} H_kv={H_kv}")
    assert _device_status()[0] == 0
