"""The float32 FMA path (tiny exact-check workload and variants) against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_exact_b200.workloads import make_dense, make_paged, workload
from tests._util import check_close, f64, paged_ref_per_head, to_dev

pytestmark = pytest.mark.gpu


def test_tiny_workload_dense_fp32():
    from paged_kv_cache_exact_b200 import api
    dense, _ = workload(1)
    Q, K, V = (t.cuda() for t in (dense.Q, dense.K, dense.V))
    got = api.prefill(Q, K, V, dense.causal, dense.scale).cpu()
    want = oracle.mha_ref(f64(dense.Q), f64(dense.K), f64(dense.V), False, 0.125)
    check_close(got, want, "tiny dense fp32")


def test_tiny_workload_paged_fp32_all_rows_and_decode():
    """The same K/V laid out in 16 permuted pages of 16: all 256 queries
    non-causal, and the decode of query row 255 alone."""
    from paged_kv_cache_exact_b200 import api
    dense, paged = workload(1)
    d = to_dev(paged)
    got = api.paged(d["q"], d["k"], d["v"], d["table"], d["lens"], 16, False, 0.125,
                    max_seq_len=256).cpu()
    want = oracle.mha_ref(f64(dense.Q), f64(dense.K), f64(dense.V), False, 0.125)
    check_close(got, want, "tiny paged fp32")
    q1 = d["q"][:, :, 255:256].contiguous()
    got1 = api.paged(q1, d["k"], d["v"], d["table"], d["lens"], 16, False, 0.125,
                     max_seq_len=256).cpu()
    check_close(got1, want[:, :, 255:256], "tiny paged decode row 255")


@pytest.mark.parametrize("N,d,causal", [(1, 64, True), (33, 64, True), (300, 128, True),
                                        (257, 128, False)])
def test_dense_fp32_shapes(N, d, causal):
    from paged_kv_cache_exact_b200 import api
    w = make_dense(21, 2, 3, N, d, dtype=torch.float32, causal=causal)
    got = api.prefill(w.Q.cuda(), w.K.cuda(), w.V.cuda(), causal, w.scale).cpu()
    want = oracle.mha_ref(f64(w.Q), f64(w.K), f64(w.V), causal, w.scale)
    check_close(got, want, f"dense fp32 N={N} d={d}")


@pytest.mark.parametrize("q_len", [1, 7, 64])
def test_paged_fp32_chunked_prefill_gqa(q_len):
    from paged_kv_cache_exact_b200 import api
    w = make_paged(22, [q_len + 5, 200, 64 + q_len], H=4, H_kv=2, d=64, page_size=16,
                   q_len=q_len, dtype=torch.float32)
    d = to_dev(w)
    got = api.paged(d["q"], d["k"], d["v"], d["table"], d["lens"], 16, True, w.scale,
                    max_seq_len=w.max_seq_len).cpu()
    check_close(got, paged_ref_per_head(w), f"paged fp32 q_len={q_len}")
