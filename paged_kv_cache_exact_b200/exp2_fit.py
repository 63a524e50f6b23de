"""Derive the degree-3 polynomial for 2^f, f in [-1/2, 1/2], used by the
prefill softmax (csrc/exp2_poly.cuh) for the exponentials it computes on the
FMA pipes.

Relative-error minimax by Lawson's method: weighted least squares on
Chebyshev nodes, re-weighting each node by its current error until the error
curve equioscillates.  Run: python -m paged_kv_cache_exact_b200.exp2_fit
"""

from __future__ import annotations

import numpy as np


def fit(deg: int = 3, nodes: int = 2000, iters: int = 200):
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))
    y = 2.0 ** f
    A = np.vander(f, deg + 1, increasing=True) / y[:, None]
    b = np.ones_like(f)
    w = np.ones_like(f)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(A * np.sqrt(w)[:, None], b * np.sqrt(w), rcond=None)
        e = np.abs(A @ c - 1)
        w = w * e
        w /= w.sum()
    return c.astype(np.float32)


def max_rel_error_fp32(c, n: int = 200001) -> float:
    g = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.full_like(g, c[-1])
    for cc in c[-2::-1]:
        p = (p * g + cc).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / 2.0 ** g.astype(np.float64) - 1).max())


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c3:", [repr(float(x)) for x in c])
    print("max relative error (fp32 Horner): %.3e" % max_rel_error_fp32(c))
