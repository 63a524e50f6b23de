"""paged_decode_noalloc: decode for callers that cannot allocate device memory
where they call attention (a plugin called from another runtime's enqueue hook
with no allocator, a latency-critical loop where cudaMalloc/cudaFree would
synchronise the device, a process whose device memory a pool holds in full).

It keeps its split partials in a static array inside the library instead of a
caller workspace.  Its results must match the fp64 oracle and paged_attn's,
within the bf16 tolerance the other tests use, on calls in a row that reuse
the shared array: case A (many splits per sequence), then case B (another split
plan, grouped heads), then case A again.  The third call runs over the
partials case B left behind and must give A's first output bit for bit.  This
file runs last so that a failure here never hides the others; it also passes
alone in a fresh process, where its first call does the one-time set-up of the
array's device address.
"""

import pytest
import torch

from paged_kv_cache_exact_b200.workloads import make_paged
from tests._util import BF16_ATOL, BF16_RTOL, check_close, paged_ref_per_head, to_dev

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


def _check(w, d, got, what):
    want_ws = _with_workspace(w, d)
    torch.cuda.synchronize()
    diff = (got.float() - want_ws.float()).abs()
    bound = BF16_ATOL + BF16_RTOL * want_ws.float().abs()
    assert bool((diff <= bound).all()), f"{what}: max diff vs paged_attn {float(diff.max()):.3e}"
    check_close(got, paged_ref_per_head(w), what)


def test_no_alloc_matches_oracle_and_workspace_path_on_calls_in_a_row():
    from paged_kv_cache_exact_b200 import binding as B
    # A: many splits per sequence (MHA, 16-token pages); B: another split plan
    # (grouped heads 8/2, 256-token pages) over the same shared array.
    wa = make_paged(81, [5000, 700, 8192, 33], H=32, H_kv=32, d=128, page_size=16, q_len=1)
    wb = make_paged(82, [600, 20000, 1, 3000], H=8, H_kv=2, d=128, page_size=256, q_len=1)
    da, db = to_dev(wa), to_dev(wb)

    first = _no_alloc(wa, da)
    torch.cuda.synchronize()
    _check(wa, da, first, "case A, first call")

    second = _no_alloc(wb, db)
    torch.cuda.synchronize()
    _check(wb, db, second, "case B")

    third = _no_alloc(wa, da)
    torch.cuda.synchronize()
    assert torch.equal(third.view(torch.int16), first.view(torch.int16)), \
        "case A after case B differs from case A's first call"

    st, bits = B.pkv_last_device_error()
    assert st == B.PKV_OK, f"device error word {bits:#x}"
