"""ctypes binding of ``libpkv.so`` (argument marshalling only).

The functions carry the names and argument order of the C ABI in
``include/pkv.h``.  Pointer arguments accept a plain integer address or any
object with ``data_ptr()`` (e.g. a torch tensor); ``stream`` accepts a
``cudaStream_t`` integer, an object with ``cuda_stream``, or None for torch's
current stream on the current device.  A non-zero status raises ``PkvError``.

There is no fallback: if the shared library is missing, importing this module
raises ImportError (build it with ``python -m paged_kv_cache_exact_b200.build``).
"""

from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "pkv.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m paged_kv_cache_exact_b200.build` (no fallback exists)")

_lib = ctypes.CDLL(LIB_PATH)

PKV_OK, PKV_ERR_INVALID_ARG, PKV_ERR_UNSUPPORTED, PKV_ERR_CUDA = 0, 1, 2, 3
PKV_ERR_TIMEOUT, PKV_ERR_BAD_TABLE, PKV_ERR_WORKSPACE, PKV_ERR_OUT_OF_PAGES = 4, 5, 6, 7
PKV_F32, PKV_BF16 = 0, 1
PKV_DEVERR_BAD_PAGE, PKV_DEVERR_BAD_LEN, PKV_DEVERR_TIMEOUT = 0x1, 0x2, 0x4
PKV_NOALLOC_SCRATCH_BYTES = 64 << 20

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

_lib.attn_prefill.restype = _i
_lib.attn_prefill.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _vp]
_lib.pkv_test_prefill_stalled.restype = _i
_lib.pkv_test_prefill_stalled.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i,
                                          _vp]
_lib.attn_prefill_fp8qk.restype = _i
_lib.attn_prefill_fp8qk.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _f, _vp]
_lib.paged_attn_workspace_size.restype = _sz
_lib.paged_attn_workspace_size.argtypes = [_i, _i, _i, _i, _i]
_lib.paged_attn.restype = _i
_lib.paged_attn.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                            _i, _f, _i, _vp, _vp, _sz, _vp]
_lib.paged_decode_noalloc.restype = _i
_lib.paged_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                      _f, _vp, _vp]
_lib.paged_kv_append.restype = _i
_lib.paged_kv_append.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp]
_lib.paged_kv_copy_pages.restype = _i
_lib.paged_kv_copy_pages.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
_i32p = ctypes.POINTER(ctypes.c_int32)
_lib.pkv_alloc_create.restype = _vp
_lib.pkv_alloc_create.argtypes = [_i, _i, _i]
_lib.pkv_alloc_destroy.restype = None
_lib.pkv_alloc_destroy.argtypes = [_vp]
_lib.pkv_alloc_add_seq.restype = _i
_lib.pkv_alloc_add_seq.argtypes = [_vp, _i]
_lib.pkv_alloc_reserve.restype = _i
_lib.pkv_alloc_reserve.argtypes = [_vp, _i, _i, _i32p, _i32p, _i32p, ctypes.POINTER(_i)]
_lib.pkv_alloc_fork.restype = _i
_lib.pkv_alloc_fork.argtypes = [_vp, _i, _i]
_lib.pkv_alloc_free_seq.restype = _i
_lib.pkv_alloc_free_seq.argtypes = [_vp, _i]
_lib.pkv_alloc_seq_len.restype = _i
_lib.pkv_alloc_seq_len.argtypes = [_vp, _i, ctypes.POINTER(_i)]
_lib.pkv_alloc_block_table.restype = _i
_lib.pkv_alloc_block_table.argtypes = [_vp, ctypes.POINTER(_i), _i, _i32p, _i32p]
_lib.pkv_alloc_num_free.restype = _i
_lib.pkv_alloc_num_free.argtypes = [_vp]
_lib.pkv_alloc_page_refs.restype = _i
_lib.pkv_alloc_page_refs.argtypes = [_vp, _i]
_lib.pkv_resolve.restype = _i
_lib.pkv_resolve.argtypes = [ctypes.POINTER(ctypes.c_int32), _i, _i, _i,
                             ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
_lib.pkv_last_device_error.restype = _i
_lib.pkv_last_device_error.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint)]
_lib.pkv_status_string.restype = ctypes.c_char_p
_lib.pkv_status_string.argtypes = [_i]


class PkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {pkv_status_string(status)} (status {status})")
        self.status = status


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn, status):
    if status != PKV_OK:
        raise PkvError(fn, status)


def pkv_status_string(status: int) -> str:
    return _lib.pkv_status_string(status).decode()


def attn_prefill(Q, K, V, O, B, H, N, d, causal, scale, dtype, stream=None):
    _check("attn_prefill", _lib.attn_prefill(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), B, H, N, d,
                                             int(causal), float(scale), dtype, _stream(stream)))


def pkv_test_prefill_stalled(Q, K, V, O, B, H, N, d, causal, scale, stall_tile, wait_limit_us,
                             stream=None):
    _check("pkv_test_prefill_stalled", _lib.pkv_test_prefill_stalled(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(O), B, H, N, d, int(causal), float(scale),
        int(stall_tile), int(wait_limit_us), _stream(stream)))


def attn_prefill_fp8qk(Q8, K8, V, O, B, H, N, d, causal, scale, q_descale, k_descale,
                       stream=None):
    _check("attn_prefill_fp8qk", _lib.attn_prefill_fp8qk(
        _ptr(Q8), _ptr(K8), _ptr(V), _ptr(O), B, H, N, d, int(causal), float(scale),
        float(q_descale), float(k_descale), _stream(stream)))


def paged_attn_workspace_size(num_seqs, H, d, max_seq_len, page_size) -> int:
    return _lib.paged_attn_workspace_size(num_seqs, H, d, max_seq_len, page_size)


def paged_attn(q, k_pages, v_pages, block_table, seq_lens, page_size, num_seqs, q_len, H, H_kv,
               d, num_pages, max_pages_per_seq, max_seq_len, causal, scale, dtype, out,
               workspace, workspace_bytes, stream=None):
    _check("paged_attn", _lib.paged_attn(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), page_size,
        num_seqs, q_len, H, H_kv, d, num_pages, max_pages_per_seq, max_seq_len, int(causal),
        float(scale), dtype, _ptr(out), _ptr(workspace), workspace_bytes, _stream(stream)))


def paged_decode_noalloc(q, k_pages, v_pages, block_table, seq_lens, page_size, num_seqs, H,
                         H_kv, d, num_pages, max_pages_per_seq, max_seq_len, scale, out,
                         stream=None):
    """Decode with the library's static scratch (allocates nothing)."""
    _check("paged_decode_noalloc", _lib.paged_decode_noalloc(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), page_size,
        num_seqs, H, H_kv, d, num_pages, max_pages_per_seq, max_seq_len, float(scale), _ptr(out),
        _stream(stream)))


def paged_kv_append(k_new, v_new, cu_new, start_pos, block_table, max_pages_per_seq, num_seqs,
                    num_new, k_pages, v_pages, num_pages, page_size, H_kv, d, dtype, stream=None):
    _check("paged_kv_append", _lib.paged_kv_append(
        _ptr(k_new), _ptr(v_new), _ptr(cu_new), _ptr(start_pos), _ptr(block_table),
        max_pages_per_seq, num_seqs, num_new, _ptr(k_pages), _ptr(v_pages), num_pages,
        page_size, H_kv, d, dtype, _stream(stream)))


def paged_kv_copy_pages(k_pages, v_pages, src, dst, n, num_pages, page_size, H_kv, d, dtype,
                        stream=None):
    _check("paged_kv_copy_pages", _lib.paged_kv_copy_pages(
        _ptr(k_pages), _ptr(v_pages), _ptr(src), _ptr(dst), n, num_pages, page_size, H_kv, d,
        dtype, _stream(stream)))


class PageAllocator:
    """The library's host page allocator (pkv_alloc_*), one object per pool."""

    def __init__(self, num_pages: int, page_size: int, max_pages_per_seq: int):
        self._h = _lib.pkv_alloc_create(num_pages, page_size, max_pages_per_seq)
        if not self._h:
            raise PkvError("pkv_alloc_create", PKV_ERR_INVALID_ARG)
        self.num_pages, self.page_size, self.max_pages = num_pages, page_size, max_pages_per_seq

    def close(self):
        if self._h:
            _lib.pkv_alloc_destroy(self._h)
            self._h = None

    __del__ = close

    def add_seq(self, seq_id: int):
        _check("pkv_alloc_add_seq", _lib.pkv_alloc_add_seq(self._h, seq_id))

    def reserve(self, seq_id: int, n_tokens: int):
        """Returns (start_pos, cow) with cow = (src, dst) or None."""
        start, src, dst, n = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int()
        _check("pkv_alloc_reserve", _lib.pkv_alloc_reserve(
            self._h, seq_id, n_tokens, ctypes.byref(start), ctypes.byref(src), ctypes.byref(dst),
            ctypes.byref(n)))
        return start.value, ((src.value, dst.value) if n.value else None)

    def fork(self, parent: int, child: int):
        _check("pkv_alloc_fork", _lib.pkv_alloc_fork(self._h, parent, child))

    def free_seq(self, seq_id: int):
        _check("pkv_alloc_free_seq", _lib.pkv_alloc_free_seq(self._h, seq_id))

    def seq_len(self, seq_id: int) -> int:
        n = ctypes.c_int()
        _check("pkv_alloc_seq_len", _lib.pkv_alloc_seq_len(self._h, seq_id, ctypes.byref(n)))
        return n.value

    def block_table(self, seq_ids):
        """Returns (table rows as lists, -1 padded; seq_lens list)."""
        n = len(seq_ids)
        ids = (ctypes.c_int * max(n, 1))(*seq_ids)
        table = (ctypes.c_int32 * max(n * self.max_pages, 1))()
        lens = (ctypes.c_int32 * max(n, 1))()
        _check("pkv_alloc_block_table", _lib.pkv_alloc_block_table(self._h, ids, n, table, lens))
        rows = [list(table[i * self.max_pages:(i + 1) * self.max_pages]) for i in range(n)]
        return rows, list(lens[:n])

    def num_free(self) -> int:
        return _lib.pkv_alloc_num_free(self._h)

    def page_refs(self, page: int) -> int:
        return _lib.pkv_alloc_page_refs(self._h, page)


def pkv_resolve(block_table_row, page_size: int, token: int):
    """Host resolution: returns (physical page, offset)."""
    row = (ctypes.c_int32 * len(block_table_row))(*[int(x) for x in block_table_row])
    phys, off = ctypes.c_int32(), ctypes.c_int32()
    _check("pkv_resolve", _lib.pkv_resolve(row, len(block_table_row), page_size, token,
                                           ctypes.byref(phys), ctypes.byref(off)))
    return phys.value, off.value


def pkv_last_device_error(stream=None):
    """Returns (status, bits) and clears the device error word."""
    bits = ctypes.c_uint(0)
    st = _lib.pkv_last_device_error(_stream(stream), ctypes.byref(bits))
    return st, bits.value


def raw_status(fn_name: str, *args) -> int:
    """Call a C entry point with raw arguments and return its status (tests)."""
    return getattr(_lib, fn_name)(*args)


def declared_functions() -> list[str]:
    """Names of the functions include/pkv.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return re.findall(r"PKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
