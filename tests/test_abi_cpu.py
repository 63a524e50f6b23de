"""The C-ABI library on a machine without a GPU: it loads, exports every
declared symbol, resolves pages on the host, and rejects bad arguments before
touching CUDA (no compute call is made here)."""

import ctypes
import math
import os

import pytest

from paged_kv_cache_exact_b200 import binding as B

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_mapping.txt")


def test_every_declared_symbol_is_exported():
    names = B.declared_functions()
    assert set(names) >= {"attn_prefill", "paged_attn", "paged_attn_workspace_size",
                          "pkv_resolve", "pkv_last_device_error", "pkv_status_string"}
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_resolve_matches_the_worked_example():
    with open(GOLDEN) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for kind, ps, table, token, *exp in rows:
        if kind != "resolve":
            continue
        e = dict(x.split("=") for x in exp)
        phys, off = B.pkv_resolve([int(x) for x in table.split(",")], int(ps), int(token))
        assert (phys, off) == (int(e["physical"]), int(e["offset"]))


def test_resolve_every_token_and_bounds():
    table = [5, 1, 9]
    for t in range(3 * 256):
        assert B.pkv_resolve(table, 256, t) == (table[t // 256], t % 256)
    with pytest.raises(B.PkvError) as ei:
        B.pkv_resolve(table, 256, 3 * 256)
    assert ei.value.status == B.PKV_ERR_INVALID_ARG


def test_status_strings():
    for s in range(7):
        assert B.pkv_status_string(s) and B.pkv_status_string(s) != "unknown status"
    assert B.pkv_status_string(99) == "unknown status"


def test_workspace_size_plan():
    # one split per sequence: no workspace
    assert B.paged_attn_workspace_size(256, 32, 128, 200, 16) == 0
    # the two decode workloads need one; the size covers (O, max, sum) per split
    for S, L, ps in [(64, 8192, 16), (16, 32768, 256)]:
        n = B.paged_attn_workspace_size(S, 32, 128, L, ps)
        assert n > 0 and n >= S * 32 * 2 * (128 + 2) * 4
        assert n == B.paged_attn_workspace_size(S, 32, 128, L, ps)   # deterministic
    assert B.paged_attn_workspace_size(0, 32, 128, 8192, 16) == 0
    assert B.paged_attn_workspace_size(4, 32, 128, 8192, 24) == 0


FAKE = 1 << 20    # aligned non-null address; never dereferenced on these paths


def _paged(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, table=FAKE, lens=FAKE, ps=16, S=2, q_len=1, H=4, H_kv=4,
             d=128, P=8, maxp=4, max_len=64, causal=1, scale=0.1, dtype=B.PKV_BF16, out=FAKE,
             ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return B.raw_status("paged_attn", a["q"], a["k"], a["v"], a["table"], a["lens"], a["ps"],
                        a["S"], a["q_len"], a["H"], a["H_kv"], a["d"], a["P"], a["maxp"],
                        a["max_len"], a["causal"], ctypes.c_float(a["scale"]), a["dtype"],
                        a["out"], a["ws"], ctypes.c_size_t(a["ws_bytes"]), a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), B.PKV_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), B.PKV_ERR_INVALID_ARG),            # misaligned
    (dict(table=FAKE + 2), B.PKV_ERR_INVALID_ARG),
    (dict(ps=8), B.PKV_ERR_INVALID_ARG),
    (dict(ps=48), B.PKV_ERR_INVALID_ARG),
    (dict(ps=512), B.PKV_ERR_INVALID_ARG),
    (dict(H=6, H_kv=4), B.PKV_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.PKV_ERR_INVALID_ARG),
    (dict(scale=0.0), B.PKV_ERR_INVALID_ARG),
    (dict(causal=2), B.PKV_ERR_INVALID_ARG),
    (dict(maxp=2, max_len=64), B.PKV_ERR_INVALID_ARG),    # table cannot hold max_len tokens
    (dict(q_len=65), B.PKV_ERR_INVALID_ARG),              # max_len < q_len
    (dict(d=96), B.PKV_ERR_UNSUPPORTED),
    (dict(dtype=7), B.PKV_ERR_INVALID_ARG),
    (dict(max_len=8192, maxp=512, ws=None, ws_bytes=0), B.PKV_ERR_WORKSPACE),
    (dict(max_len=8192, maxp=512, ws_bytes=1024), B.PKV_ERR_WORKSPACE),
    (dict(max_len=8192, maxp=512, ws=FAKE + 16), B.PKV_ERR_WORKSPACE),  # not 256-aligned
])
def test_paged_attn_rejects_bad_arguments(kw, status):
    assert _paged(**kw) == status


@pytest.mark.parametrize("args,status", [
    ((None, FAKE, FAKE, FAKE, 1, 1, 16, 128, 1, 0.1, B.PKV_BF16), B.PKV_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE + 4, 1, 1, 16, 128, 1, 0.1, B.PKV_BF16), B.PKV_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, 0, 1, 16, 128, 1, 0.1, B.PKV_BF16), B.PKV_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 128, 1, 0.1, B.PKV_BF16), B.PKV_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, 1, 0.1, B.PKV_BF16), B.PKV_ERR_UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 96, 1, 0.1, B.PKV_F32), B.PKV_ERR_UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 128, 1, math.inf, B.PKV_BF16), B.PKV_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 128, 1, 0.1, 5), B.PKV_ERR_INVALID_ARG),
])
def test_attn_prefill_rejects_bad_arguments(args, status):
    *ptrs, Bn, H, N, d, causal, scale, dtype = args
    assert B.raw_status("attn_prefill", *ptrs, Bn, H, N, d, causal, ctypes.c_float(scale),
                        dtype, None) == status


@pytest.mark.parametrize("stall,limit_us,d,status", [
    (-1, 1000, 128, B.PKV_ERR_INVALID_ARG),        # no tile to stall
    (2, 0, 128, B.PKV_ERR_INVALID_ARG),            # wait limit below 1 us
    (2, 10 ** 7 + 1, 128, B.PKV_ERR_INVALID_ARG),  # wait limit above 10 s
    (2, 1000, 64, B.PKV_ERR_UNSUPPORTED),
])
def test_stalled_prefill_hook_rejects_bad_arguments(stall, limit_us, d, status):
    """The failure-path test hook validates like attn_prefill, plus its own
    two arguments, before anything is launched."""
    assert B.raw_status("pkv_test_prefill_stalled", FAKE, FAKE, FAKE, FAKE, 1, 1, 256, d, 1,
                        ctypes.c_float(0.1), stall, limit_us, None) == status


def test_no_alloc_decode_rejects_plans_beyond_its_scratch():
    """A plan whose partials exceed PKV_NOALLOC_SCRATCH_BYTES is refused with
    PKV_ERR_WORKSPACE before anything is launched."""
    S, H, L, ps = 2048, 32, 8192, 16
    assert B.paged_attn_workspace_size(S, H, 128, L, ps) > B.PKV_NOALLOC_SCRATCH_BYTES
    st = B.raw_status("paged_decode_noalloc", FAKE, FAKE, FAKE, FAKE, FAKE, ps, S, H, H, 128,
                      1 << 16, L // ps, L, ctypes.c_float(0.1), FAKE, None)
    assert st == B.PKV_ERR_WORKSPACE
    st = B.raw_status("paged_decode_noalloc", FAKE, FAKE, FAKE, FAKE, FAKE, ps, 4, H, H, 64,
                      64, L // ps, L, ctypes.c_float(0.1), FAKE, None)
    assert st == B.PKV_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,status", [
    (dict(Q8=None), B.PKV_ERR_INVALID_ARG),
    (dict(K8=FAKE + 4), B.PKV_ERR_INVALID_ARG),           # misaligned
    (dict(B=0), B.PKV_ERR_INVALID_ARG),
    (dict(causal=2), B.PKV_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.PKV_ERR_INVALID_ARG),
    (dict(q_descale=0.0), B.PKV_ERR_INVALID_ARG),
    (dict(k_descale=math.inf), B.PKV_ERR_INVALID_ARG),
    (dict(k_descale=-1.0), B.PKV_ERR_INVALID_ARG),
    (dict(d=64), B.PKV_ERR_UNSUPPORTED),
    (dict(B=70000), B.PKV_ERR_UNSUPPORTED),
])
def test_fp8_prefill_rejects_bad_arguments(kw, status):
    a = dict(Q8=FAKE, K8=FAKE, V=FAKE, O=FAKE, B=1, H=1, N=16, d=128, causal=1, scale=0.1,
             q_descale=0.01, k_descale=0.01)
    a.update(kw)
    st = B.raw_status("attn_prefill_fp8qk", a["Q8"], a["K8"], a["V"], a["O"], a["B"], a["H"],
                      a["N"], a["d"], a["causal"], ctypes.c_float(a["scale"]),
                      ctypes.c_float(a["q_descale"]), ctypes.c_float(a["k_descale"]), None)
    assert st == status


def _append(**kw):
    a = dict(k_new=FAKE, v_new=FAKE, cu=FAKE, start=FAKE, table=FAKE, maxp=4, S=2, num_new=3,
             k=FAKE, v=FAKE, P=8, ps=16, H_kv=4, d=128, dtype=B.PKV_BF16)
    a.update(kw)
    return B.raw_status("paged_kv_append", a["k_new"], a["v_new"], a["cu"], a["start"], a["table"],
                        a["maxp"], a["S"], a["num_new"], a["k"], a["v"], a["P"], a["ps"],
                        a["H_kv"], a["d"], a["dtype"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(num_new=-1), B.PKV_ERR_INVALID_ARG),
    (dict(S=0), B.PKV_ERR_INVALID_ARG),
    (dict(ps=8), B.PKV_ERR_INVALID_ARG),
    (dict(ps=48), B.PKV_ERR_INVALID_ARG),
    (dict(ps=512), B.PKV_ERR_INVALID_ARG),
    (dict(dtype=3), B.PKV_ERR_INVALID_ARG),
    (dict(d=96), B.PKV_ERR_UNSUPPORTED),
    (dict(k_new=FAKE + 8), B.PKV_ERR_INVALID_ARG),
    (dict(cu=FAKE + 2), B.PKV_ERR_INVALID_ARG),
    (dict(table=None), B.PKV_ERR_INVALID_ARG),
    (dict(P=1 << 24, ps=256), B.PKV_ERR_UNSUPPORTED),       # pool rows beyond 2^31
    # nothing to write: success before any pointer is looked at or anything launched
    (dict(num_new=0, k_new=None, v_new=None, cu=None, start=None, table=None), B.PKV_OK),
])
def test_append_rejects_bad_arguments(kw, status):
    assert _append(**kw) == status


def _copy(**kw):
    a = dict(k=FAKE, v=FAKE, src=FAKE, dst=FAKE, n=2, P=8, ps=16, H_kv=4, d=128, dtype=B.PKV_BF16)
    a.update(kw)
    return B.raw_status("paged_kv_copy_pages", a["k"], a["v"], a["src"], a["dst"], a["n"], a["P"],
                        a["ps"], a["H_kv"], a["d"], a["dtype"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(n=-1), B.PKV_ERR_INVALID_ARG),
    (dict(P=0), B.PKV_ERR_INVALID_ARG),
    (dict(ps=24), B.PKV_ERR_INVALID_ARG),
    (dict(dtype=9), B.PKV_ERR_INVALID_ARG),
    (dict(d=32), B.PKV_ERR_UNSUPPORTED),
    (dict(v=FAKE + 4), B.PKV_ERR_INVALID_ARG),
    (dict(src=FAKE + 1), B.PKV_ERR_INVALID_ARG),
    (dict(n=0, k=None, v=None, src=None, dst=None), B.PKV_OK),
])
def test_copy_pages_rejects_bad_arguments(kw, status):
    assert _copy(**kw) == status
