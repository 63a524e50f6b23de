"""paged_decode_noalloc: decode for callers that cannot allocate device memory
where they call attention (a plugin called from another runtime's enqueue hook
with no allocator, a latency-critical loop where cudaMalloc/cudaFree would
synchronise the device, a process whose device memory a pool holds in full).

It keeps its split partials in a static array inside the library instead of a
caller workspace.  Its results must match paged_attn's, within the bf16
tolerance the other tests use, on two calls in a row: the second call finds
the first call's partials still in the shared array and must not depend on
them.  This file runs last so that a failure here never hides the others; it
also passes alone in a fresh process, where its first call does the one-time
set-up of the array's device address.
"""

import pytest
import torch

from paged_kv_cache_exact_b200.workloads import make_paged
from tests._util import BF16_ATOL, BF16_RTOL, to_dev

pytestmark = pytest.mark.gpu


def _with_workspace(w, d):
    from paged_kv_cache_exact_b200 import api
    return api.paged(d["q"], d["k"], d["v"], d["table"], d["lens"], w.page_size, True, w.scale,
                     max_seq_len=w.max_seq_len)


def _no_alloc(w, d):
    from paged_kv_cache_exact_b200 import binding as B
    out = torch.empty_like(d["q"])
    S, H, _, dim = d["q"].shape
    B.paged_decode_noalloc(d["q"], d["k"], d["v"], d["table"], d["lens"], w.page_size, S, H,
                           d["k"].shape[2], dim, d["k"].shape[0], d["table"].shape[1],
                           w.max_seq_len, w.scale, out)
    return out


def test_no_alloc_matches_workspace_path_on_two_calls_in_a_row():
    from paged_kv_cache_exact_b200 import binding as B
    cases = [(81, [5000, 700, 8192, 33], 16, 32, 32),     # many splits per sequence
             (82, [600, 20000, 1, 3000], 256, 8, 2)]      # other plan, GQA 8/2
    for seed, lens, ps, H, H_kv in cases:
        w = make_paged(seed, lens, H=H, H_kv=H_kv, d=128, page_size=ps, q_len=1)
        d = to_dev(w)
        want = _with_workspace(w, d)
        got = _no_alloc(w, d)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        diff = (got.float() - want.float()).abs()
        bound = BF16_ATOL + BF16_RTOL * want.float().abs()
        assert bool((diff <= bound).all()), f"case {seed}: max diff {float(diff.max()):.3e}"
    st, bits = B.pkv_last_device_error()
    assert st == B.PKV_OK, f"device error word {bits:#x}"
