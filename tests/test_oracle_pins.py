"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test ties one part of ``oracle/`` to a value the pages print, a closed
form, an invariant of softmax attention, brute force on tiny inputs, or a
library special case (torch's CPU float64 scaled_dot_product_attention).
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_exact_b200 import accounting
from paged_kv_cache_exact_b200.workloads import make_paged

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def _kv(*fields):
    return {k: int(v) for k, v in (f.split("=") for f in fields)}


# ---------------------------------------------------------------------------
# 1. Worked page mapping, bit-exact (values printed on the pages)
# ---------------------------------------------------------------------------

def test_worked_mapping_resolve():
    rows = [r for r in _golden_lines("worked_mapping.txt") if r[0] == "resolve"]
    assert rows
    for _, ps, table, token, *exp in rows:
        table = [int(x) for x in table.split(",")]
        e = _kv(*exp)
        phys, off = oracle.resolve(table, int(ps), int(token))
        assert int(token) // int(ps) == e["logical"]
        assert (phys, off) == (e["physical"], e["offset"])


def test_worked_mapping_page_counts():
    rows = [r for r in _golden_lines("worked_mapping.txt") if r[0] == "pages"]
    assert len(rows) == 3
    for _, ps, _, L, *exp in rows:
        e = _kv(*exp)
        assert oracle.page_count(int(L), int(ps)) == (e["n_pages"], e["last"])


def test_gather_follows_the_worked_mapping():
    """Token 300 of the [5,1,9] sequence must come from page 1, offset 44."""
    ps, H, d = 256, 2, 4
    pages = np.zeros((10, ps, H, d))
    for p in range(10):
        for o in range(ps):
            pages[p, o, :, 0] = p
            pages[p, o, :, 1] = o
    K = oracle.gather_kv(pages, [5, 1, 9], 600, ps)
    assert K.shape == (H, 600, d)
    assert K[0, 300, 0] == 1 and K[0, 300, 1] == 44
    assert K[1, 599, 0] == 9 and K[1, 599, 1] == 599 - 512
    # every token, against the per-token resolve
    for t in range(600):
        phys, off = oracle.resolve([5, 1, 9], ps, t)
        assert (K[0, t, 0], K[0, t, 1]) == (phys, off)


# ---------------------------------------------------------------------------
# 2. Softmax rows sum to one; masked entries are exactly zero
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("q_len,kv_len,causal", [(17, 17, True), (5, 23, True), (9, 31, False)])
def test_rows_sum_to_one(q_len, kv_len, causal):
    rng = np.random.default_rng(0)
    S = rng.normal(size=(q_len, kv_len)) * 5
    mask = oracle.allowed_keys(q_len, kv_len, causal)
    P = oracle.softmax_rows(S, mask)
    assert np.all(np.abs(P.sum(axis=1) - 1) <= 1e-12)
    assert np.all(P[~mask] == 0)
    assert np.all(P[mask] > 0)


def test_mask_definition_closed_form():
    # q_len == kv_len: lower triangle; q_len == 1: all keys; q_len < kv_len: shifted.
    m = oracle.allowed_keys(4, 4, True)
    assert (m == np.tril(np.ones((4, 4), bool))).all()
    assert oracle.allowed_keys(1, 7, True).all()
    m = oracle.allowed_keys(2, 5, True)
    assert m.tolist() == [[1, 1, 1, 1, 0], [1, 1, 1, 1, 1]]
    assert oracle.allowed_keys(3, 3, False).all()


# ---------------------------------------------------------------------------
# 3. Uniform scores give the mean of the visible V rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("q_len,kv_len", [(64, 64), (16, 80)])
def test_uniform_scores_mean_of_v(q_len, kv_len):
    rng = np.random.default_rng(1)
    d = 8
    Q = np.zeros((q_len, d))
    K = rng.normal(size=(kv_len, d))
    V = rng.normal(size=(kv_len, d))
    # non-causal: the mean of all rows
    O = oracle.attention_ref(Q, K, V, causal=False, scale=0.3)
    assert np.allclose(O, V.mean(axis=0)[None, :], atol=1e-13, rtol=0)
    # causal: row i averages V[0 .. i + kv_len - q_len]
    O = oracle.attention_ref(Q, K, V, causal=True, scale=0.3)
    counts = np.arange(q_len) + (kv_len - q_len) + 1
    prefix = np.cumsum(V, axis=0)[counts - 1] / counts[:, None]
    assert np.allclose(O, prefix, atol=1e-13, rtol=0)
    if q_len == kv_len:
        assert np.array_equal(O[0], V[0])           # causal row 0 sees only key 0


# ---------------------------------------------------------------------------
# 4. Paged == contiguous after an explicit gather (bit-identical)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("ps", [4, 16])
def test_paged_equals_contiguous(ps):
    rng = np.random.default_rng(2)
    S, H, H_kv, d, q_len = 3, 4, 2, 8, 5
    lens = [37, 5, 64]
    n_pages = sum((L + ps - 1) // ps for L in lens) + 3
    perm = rng.permutation(n_pages)
    k_pages = np.full((n_pages, ps, H_kv, d), np.nan)
    v_pages = np.full((n_pages, ps, H_kv, d), np.nan)
    max_pages = max((L + ps - 1) // ps for L in lens)
    table = np.full((S, max_pages), -1)
    Ks, Vs, cur = [], [], 0
    for s, L in enumerate(lens):
        K = rng.normal(size=(H_kv, L, d))
        V = rng.normal(size=(H_kv, L, d))
        Ks.append(K), Vs.append(V)
        for t in range(L):                          # scatter token by token
            if t % ps == 0:
                table[s, t // ps] = perm[cur]
                cur += 1
            k_pages[table[s, t // ps], t % ps] = K[:, t]
            v_pages[table[s, t // ps], t % ps] = V[:, t]
    q = rng.normal(size=(S, H, q_len, d))
    for causal in (True, False):
        got = oracle.paged_attention_ref(q, k_pages, v_pages, table, lens, ps, causal, 0.35)
        for s in range(S):
            want = oracle.mha_ref(q[s][None], Ks[s][None], Vs[s][None], causal, 0.35)[0]
            assert np.array_equal(got[s], want)
            assert np.isfinite(got[s]).all()        # no NaN page or tail was read


# ---------------------------------------------------------------------------
# 5. Brute force on tiny inputs (pure-Python loops, math.exp)
# ---------------------------------------------------------------------------

def _brute(Q, K, V, causal, scale):
    q_len, kv_len, d = len(Q), len(K), len(Q[0])
    out = []
    for i in range(q_len):
        lim = i + (kv_len - q_len) if causal else kv_len - 1
        s = [sum(Q[i][c] * K[j][c] for c in range(d)) * scale for j in range(lim + 1)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        tot = sum(e)
        out.append([sum(e[j] * V[j][c] for j in range(lim + 1)) / tot for c in range(len(V[0]))])
    return np.array(out)


@pytest.mark.parametrize("q_len,kv_len,d,causal", [(7, 7, 5, True), (9, 9, 16, False),
                                                   (3, 11, 4, True), (32, 32, 8, True)])
def test_brute_force_tiny(q_len, kv_len, d, causal):
    rng = np.random.default_rng(3)
    Q = rng.normal(size=(q_len, d))
    K = rng.normal(size=(kv_len, d))
    V = rng.normal(size=(kv_len, d + 1))
    got = oracle.attention_ref(Q, K, V, causal, 0.7, row_block=4)
    want = _brute(Q.tolist(), K.tolist(), V.tolist(), causal, 0.7)
    assert np.max(np.abs(got - want)) <= 1e-12


def test_brute_force_gqa_heads():
    rng = np.random.default_rng(4)
    Q = rng.normal(size=(1, 4, 6, 4))
    K = rng.normal(size=(1, 2, 6, 4))
    V = rng.normal(size=(1, 2, 6, 4))
    got = oracle.mha_ref(Q, K, V, True, 0.5)
    for h in range(4):
        want = _brute(Q[0, h].tolist(), K[0, h // 2].tolist(), V[0, h // 2].tolist(), True, 0.5)
        assert np.max(np.abs(got[0, h] - want)) <= 1e-12


# ---------------------------------------------------------------------------
# 6. Library special case: torch CPU float64 SDPA
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,d,causal", [(256, 64, False), (300, 128, True)])
def test_matches_torch_sdpa_float64(N, d, causal):
    g = torch.Generator().manual_seed(5)
    Q = torch.randn(1, 2, N, d, generator=g, dtype=torch.float64)
    K = torch.randn(1, 2, N, d, generator=g, dtype=torch.float64)
    V = torch.randn(1, 2, N, d, generator=g, dtype=torch.float64)
    want = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=causal,
                                                            scale=d ** -0.5).numpy()
    got = oracle.mha_ref(Q.numpy(), K.numpy(), V.numpy(), causal, d ** -0.5)
    assert np.max(np.abs(got - want)) <= 1e-10


def test_matches_torch_sdpa_bottom_right_mask():
    g = torch.Generator().manual_seed(6)
    q_len, kv_len, d = 40, 100, 32
    Q = torch.randn(1, 1, q_len, d, generator=g, dtype=torch.float64)
    K = torch.randn(1, 1, kv_len, d, generator=g, dtype=torch.float64)
    V = torch.randn(1, 1, kv_len, d, generator=g, dtype=torch.float64)
    i = torch.arange(q_len)[:, None]
    j = torch.arange(kv_len)[None, :]
    mask = j <= i + (kv_len - q_len)
    want = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask,
                                                            scale=0.2).numpy()
    got = oracle.mha_ref(Q.numpy(), K.numpy(), V.numpy(), True, 0.2)
    assert np.max(np.abs(got - want)) <= 1e-10


# ---------------------------------------------------------------------------
# 7. Invariants
# ---------------------------------------------------------------------------

def test_key_shift_invariance():
    rng = np.random.default_rng(7)
    Q, K, V = (rng.normal(size=(20, 8)) for _ in range(3))
    u = rng.normal(size=8)
    for causal in (True, False):
        a = oracle.attention_ref(Q, K, V, causal, 0.4)
        # adding u to every key shifts row i's scores by the constant Q_i . u
        b = oracle.attention_ref(Q, K + u[None, :], V, causal, 0.4)
        assert np.max(np.abs(a - b)) <= 1e-12


def test_key_permutation_invariance_noncausal():
    rng = np.random.default_rng(8)
    Q, K, V = (rng.normal(size=(12, 6)) for _ in range(3))
    p = rng.permutation(12)
    a = oracle.attention_ref(Q, K, V, False, 0.9)
    b = oracle.attention_ref(Q, K[p], V[p], False, 0.9)
    assert np.max(np.abs(a - b)) <= 1e-12


def test_large_scores_select_argmax_row_without_overflow():
    rng = np.random.default_rng(9)
    Q, K, V = (rng.normal(size=(10, 16)) for _ in range(3))
    O = oracle.attention_ref(Q, K, V, False, 1e4)
    assert np.isfinite(O).all()
    arg = (Q @ K.T).argmax(axis=1)
    assert np.max(np.abs(O - V[arg])) <= 1e-12


def test_single_key_returns_v0():
    rng = np.random.default_rng(10)
    q = rng.normal(size=(1, 8))
    K = rng.normal(size=(1, 8))
    V = rng.normal(size=(1, 8))
    assert np.array_equal(oracle.attention_ref(q, K, V, True, 3.0), V)


# ---------------------------------------------------------------------------
# 8. The tiled online-softmax recurrence and the split-K combine reach the
#    definition exactly (up to rounding)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("tile", [1, 7, 16, 64, 200])
@pytest.mark.parametrize("causal", [True, False])
def test_online_recurrence_equals_definition(tile, causal):
    rng = np.random.default_rng(11)
    Q = rng.normal(size=(50, 16)) * 2
    K = rng.normal(size=(50, 16)) * 2
    V = rng.normal(size=(50, 16))
    a = oracle.online_softmax_attention_ref(Q, K, V, causal, 0.5, tile)
    b = oracle.attention_ref(Q, K, V, causal, 0.5)
    assert np.max(np.abs(a - b)) <= 1e-12


def test_literal_update_would_double_normalise():
    """The printed O update (scaled by l_old/l_new, then divided by l again)
    does not reproduce attention; the unnormalised reading does.  A one-tile
    pass already shows it: the literal form ends at (P~ V) / l / l."""
    rng = np.random.default_rng(12)
    Q, K, V = (rng.normal(size=(6, 4)) for _ in range(3))
    s = Q @ K.T
    P = np.exp(s - s.max(axis=1, keepdims=True))
    l = P.sum(axis=1, keepdims=True)
    literal = (P @ V) / l / l
    assert np.max(np.abs(literal - oracle.attention_ref(Q, K, V, False, 1.0))) > 1e-3
    assert np.max(np.abs((P @ V) / l - oracle.attention_ref(Q, K, V, False, 1.0))) <= 1e-12


@pytest.mark.parametrize("bounds", [[0, 100], [0, 30, 31, 100], [0, 0, 40, 40, 100]])
def test_lse_combine_equals_definition(bounds):
    rng = np.random.default_rng(13)
    q = rng.normal(size=16) * 3
    K = rng.normal(size=(100, 16))
    V = rng.normal(size=(100, 16))
    parts = [oracle.split_partial_ref(q, K, V, 0.6, lo, hi) for lo, hi in zip(bounds, bounds[1:])]
    got = oracle.lse_combine_ref(parts)
    want = oracle.attention_ref(q[None], K, V, False, 0.6)[0]
    assert np.max(np.abs(got - want)) <= 1e-12


# ---------------------------------------------------------------------------
# 9. Value decoding and the naive traffic model the pages print
# ---------------------------------------------------------------------------

def test_bf16_decoding():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x7F80, 0x4049], dtype=np.uint16)
    v = oracle.bf16_bits_to_f64(bits)
    assert v[0] == 1.0 and v[1] == -2.0 and v[2] == 0.0 and np.signbit(v[3]) and np.isposinf(v[4])
    assert v[5] == 3.140625
    assert np.isnan(oracle.bf16_bits_to_f64(np.array([0x7FC0], dtype=np.uint16)))[0]
    t = torch.randn(1000, generator=torch.Generator().manual_seed(14)).to(torch.bfloat16)
    assert np.array_equal(oracle.to_f64(t.view(torch.int16).numpy()), t.double().numpy())


def test_naive_traffic_model_reproduces_printed_figures():
    g = dict((k, int(v)) for k, v in _golden_lines("naive_traffic.txt"))
    N, d = g["N"], g["d"]
    B = accounting.naive_traffic_bytes(N, d)
    F = accounting.naive_flops(N, d)
    assert round(F / B) == g["ops_per_byte"]
    assert round(8 * N * N / 1e6) == g["s_p_term_mb"]
    assert round(8 * N * d / 1e6) == g["nd_term_mb"]
    assert round(100 * 8 * N * N / B) == g["s_p_share_percent"]


def test_allowed_pairs_counts():
    for q_len, kv_len in [(1, 9), (7, 7), (5, 12), (128, 4096)]:
        brute = int(oracle.allowed_keys(q_len, kv_len, True).sum())
        assert accounting.allowed_pairs(q_len, kv_len, True) == brute
    assert accounting.prefill_flops(4, 32, 4096, 4096, 128, True) == 4 * 128 * 128 * 4096 * 4097 // 2


# ---------------------------------------------------------------------------
# 10. The generator's poison and fixed tables (what the parity tests rely on)
# ---------------------------------------------------------------------------

def test_generator_poison_and_fixed_table():
    w = make_paged(1, [600, 300, 17], H=2, d=8, page_size=256, decoys=2,
                   fixed_tables={0: [5, 1, 9]})
    assert w.block_table[0, :3].tolist() == [5, 1, 9]
    assert not ({5, 1, 9} & set(w.block_table[1:].flatten().tolist()))
    for p in w.decoy_pages:
        assert torch.isnan(w.k_pages[p].float()).all()
    # tail of seq 0's last page (page 9) past token 600 is poisoned, the rest is not
    assert torch.isnan(w.k_pages[9, 600 - 512:].float()).all()
    assert torch.isfinite(w.k_pages[9, :600 - 512].float()).all()
    got = oracle.paged_attention_ref(w.q.view(torch.int16).numpy(), w.k_pages.view(torch.int16).numpy(),
                                     w.v_pages.view(torch.int16).numpy(), w.block_table.numpy(),
                                     w.seq_lens.numpy(), 256, True, w.scale)
    assert np.isfinite(got).all()


def test_e4m3_decoding_all_codes():
    """Every e4m3 code decodes as torch's float8_e4m3fn does (library special
    case), plus values fixed by the format: 1.0, the largest finite 448, the
    smallest subnormal 2^-9, and the two NaN codes."""
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_bits_to_f64(codes)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert got[0x38] == 1.0 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9
    assert got[0xB8] == -1.0 and np.isnan(got[0x7F]) and np.isnan(got[0xFF])
