"""Tensor-core prefill (bf16) on the GPU against the fp64 oracle: contiguous and
paged K/V, causal and not, ragged sizes, chunked (q_len < kv_len), GQA, and the
full-size workloads on sampled rows."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_exact_b200.workloads import make_dense, make_paged, workload
from tests._util import check_close, f64, np_of, paged_ref_per_head, to_dev

pytestmark = pytest.mark.gpu


def _status_ok():
    from paged_kv_cache_exact_b200 import binding as B
    st, bits = B.pkv_last_device_error()
    assert st == 0, f"device error word {bits:#x}"


def _dense(w):
    from paged_kv_cache_exact_b200 import api
    out = api.prefill(w.Q.cuda(), w.K.cuda(), w.V.cuda(), w.causal, w.scale)
    torch.cuda.synchronize()
    return out.cpu()


def _paged(w, max_seq_len=None):
    from paged_kv_cache_exact_b200 import api
    d = to_dev(w)
    out = api.paged(d["q"], d["k"], d["v"], d["table"], d["lens"], w.page_size, w.causal,
                    w.scale, max_seq_len=max_seq_len or w.max_seq_len)
    torch.cuda.synchronize()
    return out.cpu()


@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 255, 256, 257, 300, 513, 1000])
@pytest.mark.parametrize("causal", [True, False])
def test_dense_small(N, causal):
    w = make_dense(31 + N, 1, 2, N, 128, causal=causal)
    got = _dense(w)
    want = oracle.mha_ref(f64(w.Q), f64(w.K), f64(w.V), causal, w.scale)
    check_close(got, want, f"dense N={N} causal={causal}")
    _status_ok()


def test_dense_batch_heads_and_scale():
    w = make_dense(41, 3, 5, 700, 128, causal=True, scale=0.05)
    got = _dense(w)
    want = oracle.mha_ref(f64(w.Q), f64(w.K), f64(w.V), True, 0.05)
    check_close(got, want, "dense B=3 H=5")
    _status_ok()


def test_dense_large_scores_no_overflow():
    # scores far above exp's fp32 range: the running max keeps every exp <= 2^8
    w = make_dense(42, 1, 2, 384, 128, causal=True, scale=2.0)
    got = _dense(w)
    want = oracle.mha_ref(f64(w.Q), f64(w.K), f64(w.V), True, 2.0)
    check_close(got, want, "dense large scores")


@pytest.mark.parametrize("growth", [7.5, 12.0, 40.0, 100.0])
@pytest.mark.parametrize("causal", [True, False])
def test_running_max_staircase(growth, causal):
    """Key scores that climb by `growth` (log2 units) per 128-key tile, rising
    key by key, so every row's running max grows at every tile.  The kernel
    keeps a reference max per row and moves it only when a tile's max passes
    it by more than 8 (log2 units), rescaling O before any of that tile's P is
    handed to the PV product: at 7.5 the reference moves every second tile and
    P reaches about 2^7.5 in the tile between; at 12, 40 and 100 it moves at
    every tile, and at 100 the rescale factor 2^-100 leaves the earlier O and
    row sum negligible, as they are in the exact result."""
    N, d, scale = 1000, 128, 0.088
    g = torch.Generator().manual_seed(77)
    log2e = 1.4426950408889634
    c = torch.arange(N, dtype=torch.float64) * growth / 128.0 / (d * scale * log2e)
    K = (c[:, None] * torch.ones(1, d, dtype=torch.float64)).to(torch.bfloat16)
    K = K.expand(2, N, d).reshape(1, 2, N, d).contiguous()
    Q = (1.0 + 0.05 * torch.randn(1, 2, N, d, generator=g)).to(torch.bfloat16)
    V = torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16)
    from paged_kv_cache_exact_b200 import api
    got = api.prefill(Q.cuda(), K.cuda(), V.cuda(), causal, scale)
    torch.cuda.synchronize()
    want = oracle.mha_ref(f64(Q), f64(K), f64(V), causal, scale)
    check_close(got.cpu(), want, f"staircase growth={growth} causal={causal}")
    _status_ok()


@pytest.mark.slow
def test_causal_prefill_workload_sampled_rows():
    """4 x 32 x 4096 x 128 causal: every head on 40 rows spanning tile edges,
    and two heads in full."""
    w = workload(2)
    got = _dense(w)
    rows = np.array(sorted({0, 1, 127, 128, 129, 255, 256, 511, 1023, 2047, 2048, 4094, 4095} |
                           set(np.random.default_rng(2).integers(0, 4096, 27).tolist())))
    Q, K, V = np_of(w.Q), np_of(w.K), np_of(w.V)
    for b in range(4):
        want = oracle.mha_ref(Q[b:b + 1], K[b:b + 1], V[b:b + 1], True, w.scale, rows=rows)
        check_close(got[b:b + 1, :, rows], want, f"workload 2 batch {b}")
    for b, h in [(0, 0), (3, 31)]:
        want = oracle.attention_ref(Q[b, h], K[b, h], V[b, h], True, w.scale)
        check_close(got[b, h], want, f"workload 2 head ({b},{h})")
    _status_ok()


@pytest.mark.parametrize("ps", [16, 64, 128, 256])
@pytest.mark.parametrize("lens", [[200, 1000], [128, 513, 37]])
def test_paged_full_prefill(ps, lens):
    # q_len = min(lens) so every sequence has q_len <= kv_len (chunked for the longer ones)
    q_len = min(lens)
    w = make_paged(51 + ps, lens, H=2, d=128, page_size=ps, q_len=q_len, decoys=3)
    got = _paged(w)
    check_close(got, paged_ref_per_head(w), f"paged ps={ps} lens={lens}")
    _status_ok()


@pytest.mark.parametrize("causal", [True, False])
def test_paged_chunked_prefill_gqa(causal):
    w = make_paged(61, [300, 700, 1025], H=8, H_kv=2, d=128, page_size=32, q_len=300,
                   causal=causal)
    got = _paged(w)
    check_close(got, paged_ref_per_head(w), f"paged chunked gqa causal={causal}")
    _status_ok()


def test_paged_equals_contiguous_bit_identical():
    """The same K/V as a contiguous tensor, as pages in order, and as shuffled
    pages: the three results are bit-identical (same tiles, same order)."""
    from paged_kv_cache_exact_b200 import api
    N, H, ps = 640, 2, 64
    w = make_dense(71, 1, H, N, 128, causal=True)
    dense = _dense(w)
    n_pages = N // ps
    for perm in (np.arange(n_pages), np.random.default_rng(7).permutation(n_pages)):
        k_pages = torch.empty(n_pages + 2, ps, H, 128, dtype=torch.bfloat16).fill_(float("nan"))
        v_pages = k_pages.clone()
        for lp in range(n_pages):
            k_pages[perm[lp]] = w.K[0, :, lp * ps:(lp + 1) * ps].transpose(0, 1)
            v_pages[perm[lp]] = w.V[0, :, lp * ps:(lp + 1) * ps].transpose(0, 1)
        table = torch.tensor(perm, dtype=torch.int32)[None]
        out = api.paged(w.Q.cuda(), k_pages.cuda(), v_pages.cuda(), table.cuda(),
                        torch.tensor([N], dtype=torch.int32).cuda(), ps, True, w.scale,
                        max_seq_len=N).cpu()
        assert torch.equal(out.view(torch.int16), dense.view(torch.int16))


@pytest.mark.slow
def test_long_paged_prefill_workload_sampled_rows():
    """1 x 32 x 32768 x 128 causal from 128 shuffled pages of 256: every head on
    256 rows including the tile and page edges."""
    w = workload(5)
    got = _paged(w)
    rng = np.random.default_rng(5)
    fixed = [0, 1, 127, 128, 255, 256, 257, 16383, 32766, 32767]
    rows = np.array(sorted(set(fixed) | set(rng.integers(0, 32768, 246).tolist())))
    want = paged_ref_per_head(w, rows=rows)
    check_close(got[:, :, rows], want, "workload 5")
    _status_ok()


@pytest.mark.slow
def test_chunked_prefill_full_size_sampled_rows():
    """The last 512-query chunk of four 4096-token prompts (bottom-right causal:
    query i sees keys <= i + 3584), 32 heads, pages of 256: every head on 64
    sampled rows, including the first and last of the chunk."""
    w = make_paged(81, [4096] * 4, H=32, d=128, page_size=256, q_len=512, decoys=4)
    got = _paged(w)
    rows = np.array(sorted({0, 1, 127, 128, 255, 256, 510, 511} |
                           set(np.random.default_rng(81).integers(0, 512, 56).tolist())))
    check_close(got[:, :, rows], paged_ref_per_head(w, rows=rows), "chunked prefill")
    _status_ok()


def _ref_without_tokens(w, s, drop):
    """Oracle for sequence s with the tokens in `drop` left out of the keys.

    The dropped tokens lie in the cached prefix (before the q_len new tokens),
    which every query row sees, so deleting them keeps every other key's
    causal visibility: the oracle on the shortened sequence is exact."""
    L = int(w.seq_lens[s])
    assert max(drop) < L - w.q_len
    keep = np.array([t for t in range(L) if t not in set(drop)])
    table = w.block_table[s].numpy().copy()
    table[table >= w.k_pages.shape[0]] = 0        # any page: its tokens are dropped below
    K = oracle.gather_kv(np_of(w.k_pages), table, L, w.page_size)[:, keep]
    V = oracle.gather_kv(np_of(w.v_pages), table, L, w.page_size)[:, keep]
    q = oracle.to_f64(np_of(w.q[s]))
    H, H_kv = w.q.shape[1], w.k_pages.shape[2]
    return np.stack([oracle.attention_ref(q[h], K[h // (H // H_kv)], V[h // (H // H_kv)],
                                          True, w.scale) for h in range(H)])


@pytest.mark.parametrize("ps,lens,q_len,bad_page", [(16, [400, 517], 100, 3),
                                                    (256, [700, 900], 200, 1)])
def test_paged_prefill_bad_page_is_left_out_and_flagged(ps, lens, q_len, bad_page):
    """A page id outside the pool in sequence 1's table: nothing outside the
    pool is read, the error is flagged, sequence 0 is untouched, and sequence 1
    is attention over its other keys (the bad page's keys left out, as the
    decode kernel does)."""
    from paged_kv_cache_exact_b200 import binding as B
    w = make_paged(91 + ps, lens, H=2, d=128, page_size=ps, q_len=q_len, decoys=2)
    B.pkv_last_device_error()                                  # clear
    w.block_table[1, bad_page] = w.k_pages.shape[0] + 7        # out of range
    got = _paged(w)
    st, bits = B.pkv_last_device_error()
    assert st == B.PKV_ERR_BAD_TABLE and bits & B.PKV_DEVERR_BAD_PAGE, (st, bits)
    check_close(got[:1], paged_ref_per_head(w, seqs=[0]), "good sequence")
    drop = list(range(bad_page * ps, (bad_page + 1) * ps))
    check_close(got[1], _ref_without_tokens(w, 1, drop), "sequence with a bad page")


def test_bounded_wait_runs_out_then_the_next_call_is_correct():
    """The failure path of the prefill pipeline, without faulting or hanging
    the GPU: with every wait bounded at 1 ms and one K load never issued, the
    CTAs waiting for it give up, drain what they issued, free their tensor
    memory and exit; the device error word says PKV_ERR_TIMEOUT.  The next
    normal call on the same context is correct against the oracle."""
    from paged_kv_cache_exact_b200 import api
    from paged_kv_cache_exact_b200 import binding as B
    w = make_dense(95, 1, 2, 1024, 128, causal=True)
    Q, K, V = w.Q.cuda(), w.K.cuda(), w.V.cuda()
    O = torch.empty_like(Q)
    B.pkv_last_device_error()                                  # clear
    B.pkv_test_prefill_stalled(Q, K, V, O, 1, 2, 1024, 128, True, w.scale, 2, 1000)
    torch.cuda.synchronize()
    st, bits = B.pkv_last_device_error()
    assert st == B.PKV_ERR_TIMEOUT and bits & B.PKV_DEVERR_TIMEOUT, (st, bits)
    got = api.prefill(Q, K, V, True, w.scale).cpu()
    check_close(got, oracle.mha_ref(f64(w.Q), f64(w.K), f64(w.V), True, w.scale),
                "prefill after a timed-out call")
    _status_ok()
