"""Exact attention over contiguous and paged K/V for B200 (sm_100a).

The compute path is the C ABI in ``include/pkv.h`` implemented by
``libpkv.so`` (hand-written CUDA for sm_100a); ``binding`` marshals Python
arguments to it.  PyTorch is only used by callers for device memory and
streams.  Importing ``binding`` fails loudly when the library is not built.
"""

__all__ = ["binding", "workloads", "accounting", "build"]
