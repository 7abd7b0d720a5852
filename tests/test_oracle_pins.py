"""Pins of the fp64 oracle to things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle (a dropped head, a
wrong sign or index, a transposed operand, an off-by-one window, a wrong tie
order, a wrong FP8 rounding) fails at least one of them:

* library special cases: torch's fp64 scaled_dot_product_attention (causal and
  masked), torch.topk, torch.matmul, torch's float8_e4m3fn codec;
* closed forms: uniform attention (K = 0), the forced window, the KV bytes the
  method's results table prints;
* brute force: every k-subset of the candidates on tiny rows;
* invariants the pages fix: sum of the head-summed probabilities = H, sparse
  equals dense attention when the budget covers the prefix, planted needles are
  selected in their target rows.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


def _sdpa(q, K, V, mask=None, causal=False):
    """torch fp64 SDPA with the single KV head broadcast to every query head.
    q: [T, H, d] -> out [T, H, dv]."""
    qt = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))      # H,T,d
    H = qt.shape[0]
    kt = torch.from_numpy(K)[None].expand(H, -1, -1)
    vt = torch.from_numpy(V)[None].expand(H, -1, -1)
    m = None if mask is None else torch.from_numpy(mask)[None].expand(H, -1, -1)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, is_causal=causal)
    return o.numpy().transpose(1, 0, 2)


# ---------------------------------------------------------------- FP8 codec

def test_e4m3_decode_exhaustive_against_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes.numpy())
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2                      # 0x7F and 0xFF only
    assert np.array_equal(ref[~nan], got[~nan])
    assert oracle.E4M3_TABLE[0x7E] == 448.0


def test_e4m3_encode_against_torch_cast():
    g = np.random.default_rng(1)
    vals = np.concatenate([
        g.uniform(-448, 448, 20000), g.uniform(-1, 1, 20000),
        g.uniform(-2 ** -6, 2 ** -6, 5000),
        # exact midpoints between neighbouring codes: ties go to the even code
        (oracle._POS_VALUES[1:] + oracle._POS_VALUES[:-1]) / 2,
        -(oracle._POS_VALUES[1:] + oracle._POS_VALUES[:-1]) / 2,
        oracle._POS_VALUES, [0.0, -0.0, 448.0, -448.0],
    ]).astype(np.float32)            # torch casts from fp32; all are exact fp32
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(vals.astype(np.float64))
    assert np.array_equal(ref, got)


def test_e4m3_encode_saturates():
    x = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e6, -1e30])
    got = oracle.e4m3_decode(oracle.e4m3_encode(x))
    assert np.array_equal(got, [448, 448, 448, 448, 448, 448, -448])


def test_quantize_rows_bounds_and_zero_row():
    X = _rand((64, 256), 2)
    X[3] = 0.0
    codes, scale, y = oracle.quantize_rows_e4m3(X)
    amax = np.abs(X).max(1)
    assert scale[3] == 1.0 and np.all(codes[3] == 0)
    nz = amax > 0
    assert np.allclose(scale[nz], amax[nz] / 448.0, rtol=0, atol=0)
    # every row reaches +-448 at its amax element, and the error is within half
    # an E4M3 ulp (2^-4 relative for normals, 2^-10 absolute for subnormals)
    deq = oracle.e4m3_decode(codes)
    assert np.all(np.abs(deq[nz]).max(1) == 448.0)
    err = np.abs(deq - y)
    bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10)
    assert np.all(err <= bound + 1e-12)


# ---------------------------------------------------------------- bridging

def test_bridge_matches_torch_matmul():
    h = _rand((37, 64), 3)
    W = _rand((24, 64), 4)
    ref = torch.matmul(torch.from_numpy(h), torch.from_numpy(W).T).numpy()
    assert np.allclose(oracle.bridge_rows(h, W), ref, rtol=1e-13, atol=1e-12)
    # a transposed projection would not even have the right shape here
    assert oracle.bridge_rows(h, W).shape == (37, 24)


# ---------------------------------------------------------------- full attention

@pytest.mark.parametrize("T,H,d,q_start", [(40, 4, 16, 0), (33, 3, 8, 0), (20, 2, 8, 11)])
def test_full_output_matches_sdpa(T, H, d, q_start):
    kv = q_start + T
    q = _rand((T, H, d), 5)
    K = _rand((kv, d), 6)
    V = _rand((kv, d), 7)
    rows = oracle.full_attn_select(q, K, V, range(T), q_start, window=4, topk=3)
    mask = np.tril(np.ones((T, kv), dtype=bool), k=q_start)
    ref = _sdpa(q, K, V, mask=mask)
    for t in range(T):
        assert np.allclose(rows[t].O, ref[t], rtol=1e-12, atol=1e-12)


def test_sigma_matches_sdpa_probability_rows():
    """With V = identity the attention output of head h is its probability row,
    so the head sum of SDPA's output is the selection score."""
    T, H, d = 30, 5, 8
    q = _rand((T, H, d), 8)
    K = _rand((T, d), 9)
    probs = _sdpa(q, K, np.eye(T), causal=True)               # [T, H, T]
    rows = oracle.full_attn_select(q, K, np.zeros((T, 1)), range(T), 0, 4, 3)
    for t in range(T):
        assert np.allclose(rows[t].sigma, probs[t].sum(0)[:t + 1], rtol=1e-12, atol=1e-14)
        assert np.allclose(probs[t].sum(0)[t + 1:], 0)


def test_sigma_sums_to_H():
    T, H, d = 50, 6, 16
    rows = oracle.full_attn_select(_rand((T, H, d), 10), _rand((T, d), 11),
                                   _rand((T, d), 12), range(T), 0, 8, 5)
    for r in rows.values():
        assert abs(r.sigma.sum() - H) < 1e-12


def test_uniform_attention_closed_form():
    """K = 0: every logit is 0, P = 1/(p+1), sigma = H/(p+1) for every key, the
    output is the mean of the visible V rows, and with all scores tied the
    selection is the k smallest positions."""
    T, H, d, W, k = 60, 4, 8, 8, 10
    V = _rand((T, d), 13)
    rows = oracle.full_attn_select(_rand((T, H, d), 14), np.zeros((T, d)), V,
                                   range(T), 0, W, k)
    for t, r in rows.items():
        assert np.allclose(r.sigma, H / (t + 1), rtol=1e-14)
        assert np.allclose(r.O, np.broadcast_to(V[:t + 1].mean(0), (H, d)), atol=1e-13)
        n_cand = max(0, t - W + 1)
        n_sel = min(k, n_cand)
        assert list(r.idx[W:W + n_sel]) == list(range(n_sel))


@pytest.mark.parametrize("p,W,k", [(0, 128, 1024), (5, 128, 1024), (127, 128, 1024),
                                   (128, 128, 1024), (1151, 128, 1024), (1152, 128, 1024),
                                   (5000, 128, 1024), (30, 4, 3), (3, 4, 3), (4, 4, 3)])
def test_window_and_padding_closed_form(p, W, k):
    d = 4
    K = _rand((p + 1, d), 15)
    r = oracle.select_row(_rand((2, d), 16), K, K, p, W, k, 0.5)
    expect_win = [x if x >= 0 else -1 for x in range(p - W + 1, p + 1)]
    assert list(r.idx[:W]) == expect_win
    n_cand = max(0, p - W + 1)
    n_sel = min(k, n_cand)
    assert r.n_sel == n_sel
    assert np.all(r.idx[W + n_sel:] == -1)
    sel = r.idx[W:W + n_sel]
    assert np.all(sel <= p - W) and np.all(np.diff(sel) > 0)
    assert r.idx.shape == (W + k,)


def test_topk_matches_torch_topk():
    T, H, d, W, k = 400, 8, 32, 16, 50
    rows = oracle.full_attn_select(_rand((T, H, d), 17), _rand((T, d), 18),
                                   _rand((T, d), 19), range(100, T, 7), 0, W, k)
    for t, r in rows.items():
        n_cand = t - W + 1
        ref = torch.topk(torch.from_numpy(r.sigma[:n_cand]), k).indices.numpy()
        assert set(ref.tolist()) == set(r.idx[W:W + k].tolist())
        assert r.tau == pytest.approx(float(np.sort(r.sigma[:n_cand])[-k]), rel=0)


def _brute_force_topk(sigma_c, k):
    """The unique k-subset whose every member outranks every non-member under
    (score, -position) order -- found by trying all subsets."""
    n = len(sigma_c)
    if n <= k:
        return tuple(range(n))
    key = [(sigma_c[j], -j) for j in range(n)]
    found = [S for S in itertools.combinations(range(n), k)
             if min(key[j] for j in S) > max(key[j] for j in range(n) if j not in S)]
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_tiny(seed):
    T, H, d, W, k = 20, 3, 4, 4, 3
    q = _rand((T, H, d), 100 + seed)
    K = _rand((T, d), 200 + seed)
    if seed % 2:                 # duplicated keys: exact score ties
        K[3] = K[1]
        K[7] = K[1]
        K[10] = K[5]
    rows = oracle.full_attn_select(q, K, _rand((T, d), 300 + seed), range(T), 0, W, k)
    for t, r in rows.items():
        n_cand = max(0, t - W + 1)
        ref = _brute_force_topk(r.sigma[:n_cand], k)
        assert tuple(r.idx[W:W + len(ref)]) == ref


def test_decode_equals_prefill_last_row():
    """A decode query at position N-1 over the dequantised cache is the last
    prefill row over the same K/V."""
    B, N, H, d = 2, 300, 4, 16
    case = synth.make_decode_case(B, N, H, d, window=16, topk=20, n_sparse=1)
    dec = oracle.decode_select(case.Q, case.Kc, case.Vc, case.ks, case.vs, range(B), N, 16, 20)
    for b in range(B):
        K = case.Kc[b].view(torch.float8_e4m3fn).to(torch.float64) * case.ks[b, :, None].double()
        V = case.Vc[b].view(torch.float8_e4m3fn).to(torch.float64) * case.vs[b, :, None].double()
        q = case.Q[b].double().numpy()
        qq = np.zeros((N, H, d))
        qq[N - 1] = q
        pre = oracle.full_attn_select(qq, K.numpy(), V.numpy(), [N - 1], 0, 16, 20)[N - 1]
        assert np.array_equal(pre.idx, dec[b].idx)
        assert np.allclose(pre.O, dec[b].O, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- sparse layers

def test_sparse_matches_masked_sdpa():
    T, H, d = 64, 4, 16
    g = np.random.default_rng(20)
    qs = _rand((T, H, d), 21)
    K = _rand((T, d), 22)
    V = _rand((T, d), 23)
    n_idx = 12
    idx = np.full((T, n_idx), -1, dtype=np.int32)
    mask = np.zeros((T, T), dtype=bool)
    for t in range(T):
        n = min(t + 1, int(g.integers(1, n_idx + 1)))
        S = np.sort(g.choice(t + 1, size=n, replace=False))
        idx[t, :n] = S
        mask[t, S] = True
    got = oracle.sparse_attn(qs, K, V, idx, range(T))
    ref = _sdpa(qs, K, V, mask=mask)
    for t in range(T):
        assert np.allclose(got[t], ref[t], rtol=1e-12, atol=1e-12)


def test_sparse_equals_dense_when_budget_covers_prefix():
    """Sparse layers read the full layer's KV: when window + topk covers the
    whole prefix, the index set is the prefix and sparse = dense causal."""
    T, H, d, W, k = 48, 4, 16, 8, 48
    case = synth.make_prefill_case(T, H, d, W, k, n_sparse=1, seed=3)
    Q, K, V = (x.double().numpy() for x in (case.Q, case.K, case.V))
    qs = case.Q_sparse[0].double().numpy()
    rows = oracle.full_attn_select(Q, K, V, range(T), 0, W, k)
    idx = np.stack([rows[t].idx for t in range(T)])
    got = oracle.sparse_attn(qs, K, V, idx, range(T))
    ref = _sdpa(qs, K, V, causal=True)
    for t in range(T):
        assert sorted(idx[t][idx[t] >= 0].tolist()) == list(range(t + 1))
        assert np.allclose(got[t], ref[t], rtol=1e-12, atol=1e-12)


def test_needles_are_selected_in_their_target_rows():
    """Token-level selection can pick an isolated key: every planted needle is in
    the selection of the row it was aligned with (workload of 1024 queries,
    8 heads, d = 128, window 128 + top-256)."""
    c = synth.CONFIGS[1]
    case = synth.make_prefill_case(c["T"], c["H"], c["d"], c["window"], c["topk"],
                                   n_sparse=0, n_needles=c["n_needles"], seed=0)
    Q, K, V = (x.double().numpy() for x in (case.Q, case.K, case.V))
    assert len(case.needles) == 4
    rows = oracle.full_attn_select(Q, K, V, [i for _, i in case.needles], 0,
                                   c["window"], c["topk"])
    for p, i in case.needles:
        assert p in set(rows[i].idx[c["window"]:].tolist())


# ---------------------------------------------------------------- printed figures

def test_kv_cache_bytes_match_the_results_table():
    """One K row and one V row of d bytes each (FP8) per token per full layer:
    the results table's KV @1M (FP8) column follows to its printed rounding."""
    g = json.load(open(os.path.join(GOLDEN, "paper_figures.json")))
    N = g["tokens_at_1m"]
    for name in ("hysparse2", "hysparse", "hybrid_swa"):
        m = g[name]
        b = m["full_layers"] * N * m["kv_heads"] * (m["d_qk"] + m["d_v"])
        assert abs(b / 1e9 - m["kv_gb_at_1m_fp8"]) <= 0.015, name
    assert g["window"] + g["topk"] == 1152


# ---------------------------------------------------------------- mutation checks

def test_pins_catch_a_dropped_head():
    """Plant a mistake in a copy of the oracle's score (one head left out) and
    check that the invariant and the SDPA pin both reject it."""
    T, H, d = 24, 4, 8
    q = _rand((T, H, d), 30)
    K = _rand((T, d), 31)
    r = oracle.select_row(q[T - 1], K, K, T - 1, 4, 3, 1 / math.sqrt(d))
    s = (q[T - 1] @ K.T) / math.sqrt(d)
    P = np.exp(s - s.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    bad = r.sigma - P[0]
    assert abs(bad.sum() - H) > 0.5
    probs = _sdpa(q, K, np.eye(T), causal=True)[T - 1].sum(0)
    assert not np.allclose(bad, probs)
    assert np.allclose(r.sigma, probs, rtol=1e-12)


def test_pins_catch_a_shifted_window():
    p, W = 300, 128
    good = oracle.window_slots(p, W)
    assert good[-1] == p and good[0] == p - W + 1
    shifted = oracle.window_slots(p - 1, W)
    assert not np.array_equal(shifted, good)
