"""attn_prefill_fp8qk: e4m3 Q and K with per-tensor descales, bf16 V and output.
The oracle computes attention on the dequantized e4m3 values, so the only
difference left is the kernel's f32 accumulation and bf16 rounding of P and O
(the same tolerance as the bf16 path)."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_exact_b200.workloads import make_dense
from tests._util import check_close, f64, np_of

pytestmark = pytest.mark.gpu


def quantize(x: torch.Tensor):
    """Per-tensor e4m3 quantization: (codes as uint8, descale)."""
    amax = float(x.float().abs().max())
    descale = amax / 448.0
    codes = (x.float() / descale).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, descale


def run_fp8(w):
    from paged_kv_cache_exact_b200 import binding as B
    Q8, qd = quantize(w.Q)
    K8, kd = quantize(w.K)
    Bn, H, N, d = w.Q.shape
    O = torch.empty_like(w.V, device="cuda")
    B.attn_prefill_fp8qk(Q8.cuda(), K8.cuda(), w.V.cuda(), O, Bn, H, N, d, w.causal, w.scale,
                         qd, kd)
    torch.cuda.synchronize()
    Qd = oracle.e4m3_bits_to_f64(Q8.numpy()) * qd
    Kd = oracle.e4m3_bits_to_f64(K8.numpy()) * kd
    return O.cpu(), Qd, Kd


@pytest.mark.parametrize("N", [1, 100, 128, 300, 1000])
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_qk_prefill_small(N, causal):
    from paged_kv_cache_exact_b200 import binding as B
    w = make_dense(111 + N, 2, 3, N, 128, causal=causal)
    got, Qd, Kd = run_fp8(w)
    want = oracle.mha_ref(Qd, Kd, f64(w.V), causal, w.scale)
    check_close(got, want, f"fp8 N={N} causal={causal}")
    assert B.pkv_last_device_error()[0] == 0


@pytest.mark.slow
def test_fp8_qk_prefill_full_size_sampled_rows():
    w = make_dense(1002, 4, 32, 4096, 128, causal=True)
    got, Qd, Kd = run_fp8(w)
    V = np_of(w.V)
    rows = np.array(sorted({0, 1, 127, 128, 2047, 4095} |
                           set(np.random.default_rng(3).integers(0, 4096, 18).tolist())))
    for b in range(4):
        want = oracle.mha_ref(Qd[b:b + 1], Kd[b:b + 1], V[b:b + 1], True, w.scale, rows=rows)
        check_close(got[b:b + 1, :, rows], want, f"fp8 full size batch {b}")
