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


@pytest.mark.parametrize("seed", range(4))
def test_tau_is_torch_topk_kth_value_with_ties(seed):
    """tau (the k-th largest candidate score, the centre of the tie margin) is
    torch.topk's last value, also on rows whose boundary falls inside a run of
    exactly tied scores (duplicated keys, and K = 0 where every score ties)."""
    T, H, d, W, k = 60, 3, 8, 4, 7
    q = _rand((T, H, d), 400 + seed)
    K = _rand((T, d), 500 + seed)
    if seed == 3:
        K[:] = 0.0                                     # every candidate score equal
    else:
        for a, b in ((0, 2), (0, 5), (0, 9), (4, 11), (4, 13), (6, 20), (6, 21), (6, 22)):
            K[b] = K[a]                                # runs of exactly equal scores
    rows = oracle.full_attn_select(q, K, _rand((T, d), 600 + seed), range(T), 0, W, k)
    n_ties = 0
    for t, r in rows.items():
        n_cand = max(0, t - W + 1)
        if n_cand <= k:
            assert r.tau is None
            continue
        sc = torch.from_numpy(r.sigma[:n_cand])
        vals = torch.topk(sc, k).values
        assert r.tau == float(vals[-1])
        # the k-th and (k+1)-th values differ unless the boundary sits in a tie run
        kp1 = float(torch.topk(sc, k + 1).values[-1])
        n_ties += r.tau == kp1
        assert r.tau >= kp1
    if seed == 3:
        assert n_ties == sum(1 for t in range(T) if t - W + 1 > k)


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


def _fp8_cache(B, N, d, seed, lo, hi):
    """Random finite E4M3 codes (the two NaN codes avoided) and per-token
    scales drawn log-uniformly in [lo, hi) -- a different range per call, so a
    K scale used for V (or the reverse) moves every output."""
    g = np.random.default_rng(seed)
    codes = g.integers(0, 0x7E, size=(B, N, d)).astype(np.uint8)
    codes |= (g.integers(0, 2, size=(B, N, d)) << 7).astype(np.uint8)      # random signs
    scales = np.exp(g.uniform(np.log(lo), np.log(hi), size=(B, N)))
    return torch.from_numpy(codes), torch.from_numpy(scales)


def _sparse_decode_ref(Qs, Kc, Vc, ks, vs, idx, b, scale):
    """torch only: dequantise sequence b's cache through torch's own E4M3 type,
    gather the slots of idx[b] (a repeated slot is gathered twice), fp64 SDPA."""
    S = torch.from_numpy(idx[b][idx[b] >= 0].astype(np.int64))
    K = Kc[b].view(torch.float8_e4m3fn).to(torch.float64) * ks[b][:, None]
    V = Vc[b].view(torch.float8_e4m3fn).to(torch.float64) * vs[b][:, None]
    q = torch.from_numpy(np.asarray(Qs[b], dtype=np.float64))[:, None, :]          # [H, 1, d]
    Kg = K.index_select(0, S)[None].expand(q.shape[0], -1, -1)
    Vg = V.index_select(0, S)[None].expand(q.shape[0], -1, -1)
    return F.scaled_dot_product_attention(q, Kg, Vg, scale=scale)[:, 0].numpy()


def test_sparse_attn_decode_matches_sdpa_over_torch_dequantised_cache():
    """The sparse decode oracle reads sequence b's own cache rows, K codes with
    K scales and V codes with V scales: checked against torch's E4M3 decode and
    fp64 SDPA over the gathered rows, with -1 slots, repeated slots, an empty
    row and per-sequence scale ranges; then two planted gather mistakes (K and
    V scales swapped, every sequence reading its neighbour's cache) must fail."""
    B, N, H, d, n_idx = 4, 90, 4, 16, 24
    Kc, ks = _fp8_cache(B, N, d, 40, 1e-3, 1e-1)
    Vc, vs = _fp8_cache(B, N, d, 41, 0.5, 8.0)
    for b in range(B):                                # per-sequence scale ranges
        ks[b] *= 3.0 ** b
        vs[b] *= 0.5 ** b
    Qs = _rand((B, H, d), 42)
    g = np.random.default_rng(43)
    idx = np.full((B, n_idx), -1, dtype=np.int32)
    for b in range(B - 1):
        n = int(g.integers(5, n_idx + 1))
        idx[b, :n] = np.sort(g.integers(0, N, size=n))     # repeats likely
        idx[b, g.random(n_idx) < 0.2] = -1
    idx[0, :3] = 17                                    # one key in three slots
    idx[1, 5] = idx[1, 6] = 40
    # sequence B-1: no valid slot -> zero output
    scale = 1 / math.sqrt(d)
    got = oracle.sparse_attn_decode(Qs, Kc, Vc, ks, vs, idx, range(B))
    for b in range(B - 1):
        assert np.allclose(got[b], _sparse_decode_ref(Qs, Kc, Vc, ks, vs, idx, b, scale), rtol=1e-12, atol=1e-12)
    assert np.array_equal(got[B - 1], np.zeros((H, d)))
    # planted mistakes in the gather, on the CPU: each moves some sequence's output far
    swapped = oracle.sparse_attn_decode(Qs, Kc, Vc, vs, ks, idx, range(B - 1))
    assert max(np.abs(swapped[b] - got[b]).max() for b in range(B - 1)) > 1e-2
    shifted = oracle.sparse_attn_decode(Qs, torch.roll(Kc, 1, 0), torch.roll(Vc, 1, 0), ks, vs, idx, range(B - 1))
    assert max(np.abs(shifted[b] - got[b]).max() for b in range(B - 1)) > 1e-2


def test_sparse_row_with_no_valid_entry_is_zero():
    q = _rand((4, 8), 44)
    K = _rand((10, 8), 45)
    V = _rand((10, 6), 46)
    out = oracle.sparse_attn_row(q, K, V, np.full(5, -1, dtype=np.int32), 0.3)
    assert out.shape == (4, 6) and np.array_equal(out, np.zeros((4, 6)))
    # one valid entry: probability 1 on that key, the output is its V row
    one = oracle.sparse_attn_row(q, K, V, np.array([-1, 7, -1], dtype=np.int32), 0.3)
    assert np.allclose(one, np.broadcast_to(V[7], (4, 6)), rtol=0, atol=1e-15)


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


# ---------------------------------------------------------------- block-level selection

def test_block_selection_with_block_1_is_token_selection():
    """Blocks of one token are tokens: the block variant's index rows equal the
    token-level rows for every query (same k), which are pinned above."""
    T, H, d, W, k = 120, 4, 16, 8, 9
    q, K, V = _rand((T, H, d), 700), _rand((T, d), 701), _rand((T, d), 702)
    tok = oracle.full_attn_select(q, K, V, range(T), 0, W, k)
    blk = oracle.full_attn_select_blocks(q, K, V, range(T), 0, W, 1, k)
    for t in range(T):
        assert np.array_equal(blk[t][1].idx, tok[t].idx)
        assert blk[t][1].tau == tok[t].tau


@pytest.mark.parametrize("seed", range(4))
def test_block_selection_brute_force_tiny(seed):
    """Every k-subset of blocks on rows of up to 40 candidates: the chosen
    blocks are the unique subset that outranks the rest under (score, -block);
    the row lists exactly their candidate positions; the scores partition the
    candidates' sigma."""
    T, H, d, W, B, k = 48, 3, 4, 4, 4, 3
    q, K = _rand((T, H, d), 800 + seed), _rand((T, d), 810 + seed)
    if seed % 2:
        K[4:8] = K[12:16]                          # two blocks with equal scores where sigma allows
    rows = oracle.full_attn_select_blocks(q, K, _rand((T, d), 820 + seed), range(T), 0, W, B, k)
    for t, (r, b) in rows.items():
        n_cand = max(0, t - W + 1)
        nb = (n_cand + B - 1) // B
        assert b.block_score.shape == (nb,)
        assert abs(b.block_score.sum() - r.sigma[:n_cand].sum()) <= 1e-12
        ref = _brute_force_topk(b.block_score, k)
        assert tuple(b.blocks.tolist()) == ref
        want = [j for c in ref for j in range(c * B, min(n_cand, (c + 1) * B))]
        n = len(want)
        assert list(b.idx[W:W + n]) == want and np.all(b.idx[W + n:] == -1)
        assert np.array_equal(b.idx[:W], oracle.window_slots(t, W))
        if nb > k:
            assert b.tau == float(torch.topk(torch.from_numpy(b.block_score), k).values[-1])


def test_block_selection_uniform_closed_form():
    """K = 0: sigma = H/(p+1) for every key, so every full block scores
    B*H/(p+1), the partial boundary block less, and with the full blocks tied
    the selection is the first k blocks."""
    T, H, d, W, B, k = 200, 4, 8, 16, 8, 5
    rows = oracle.full_attn_select_blocks(_rand((T, H, d), 830), np.zeros((T, d)), _rand((T, d), 831),
                                          range(T), 0, W, B, k)
    for t, (r, b) in rows.items():
        n_cand = max(0, t - W + 1)
        full = n_cand // B
        assert np.allclose(b.block_score[:full], B * H / (t + 1), rtol=1e-13)
        if n_cand % B:
            assert np.isclose(b.block_score[-1], (n_cand % B) * H / (t + 1), rtol=1e-13)
        nb = b.block_score.shape[0]
        expect = list(range(min(k, nb))) if full >= k or nb <= k else list(range(full)) + [nb - 1]
        assert b.blocks.tolist() == expect


# ---------------------------------------------------------------- SWA with partial RoPE

def test_rope_preserves_pair_norms_and_leaves_the_rest():
    X = _rand((7, 3, 96), 900)
    pos = np.array([0, 1, 5, 77, 1000, 65535, 262143])
    Y = oracle.rope_rows(X.transpose(1, 0, 2), pos).transpose(1, 0, 2)     # rows on axis -2
    assert np.array_equal(Y[..., 64:], X[..., 64:])                        # dims past 64 untouched
    n_x = X[..., :32] ** 2 + X[..., 32:64] ** 2
    n_y = Y[..., :32] ** 2 + Y[..., 32:64] ** 2
    assert np.allclose(n_y, n_x, rtol=1e-12)
    assert np.allclose(Y[0], X[0], rtol=0, atol=0)                          # position 0: identity


def test_rope_scores_depend_only_on_the_distance():
    """<rope(q, m), rope(k, n)> is a function of m - n: shifting both positions
    by the same amount leaves every score unchanged, and the score at distance
    0 is the plain dot product on the rotated dims."""
    q = _rand((1, 64), 901)
    k = _rand((1, 64), 902)
    for m, n in ((10, 3), (5000, 4993), (123456, 123449)):
        a = oracle.rope_rows(q, np.array([m])) @ oracle.rope_rows(k, np.array([n])).T
        b = oracle.rope_rows(q, np.array([m - n])) @ oracle.rope_rows(k, np.array([0])).T
        assert np.allclose(a, b, rtol=1e-9, atol=1e-9)
    same = oracle.rope_rows(q, np.array([777])) @ oracle.rope_rows(k, np.array([777])).T
    assert np.allclose(same, q @ k.T, rtol=1e-10)
    # a planted mistake: pairs (2i, 2i+1) instead of (i, i + 32) keep norms but
    # break the distance rule against this pairing's rotation of the same vector
    def rope_interleaved(x, p):
        inv = 10000.0 ** (-2.0 * np.arange(32) / 64)
        ang = p * inv
        y = x.copy()
        y[:, 0:64:2] = x[:, 0:64:2] * np.cos(ang) - x[:, 1:64:2] * np.sin(ang)
        y[:, 1:64:2] = x[:, 0:64:2] * np.sin(ang) + x[:, 1:64:2] * np.cos(ang)
        return y
    assert not np.allclose(rope_interleaved(q, 10), oracle.rope_rows(q, np.array([10])))


@pytest.mark.parametrize("T,W,q_start", [(70, 16, 0), (40, 8, 25), (33, 100, 0)])
def test_swa_matches_sdpa_with_a_band_mask(T, W, q_start):
    H, d = 3, 80
    kv = q_start + T
    q = _rand((T, H, d), 903)
    K = _rand((kv, d), 904)
    V = _rand((kv, d), 905)
    got = oracle.swa_attn(q, K, V, range(T), q_start, W)
    # torch: rotate with the oracle's RoPE (pinned above), then fp64 SDPA with
    # the band mask of the window
    qr = np.stack([oracle.rope_rows(q[t][None], np.array([q_start + t]))[0] for t in range(T)])
    kr = oracle.rope_rows(K, np.arange(kv))
    pos = q_start + np.arange(T)[:, None]
    key = np.arange(kv)[None, :]
    mask = (key <= pos) & (key > pos - W)
    ref = _sdpa(qr, kr, V, mask=mask)
    for t in range(T):
        assert np.allclose(got[t], ref[t], rtol=1e-12, atol=1e-12)


def test_swa_with_a_window_over_the_prefix_is_causal_attention():
    """A window at least as long as the prefix is plain causal attention over the
    rotated q and k: the same as the full-attention oracle on rotated inputs."""
    T, H, d = 50, 4, 64
    q, K, V = _rand((T, H, d), 906), _rand((T, d), 907), _rand((T, d), 908)
    got = oracle.swa_attn(q, K, V, range(T), 0, window=T)
    qr = np.stack([oracle.rope_rows(q[t][None], np.array([t]))[0] for t in range(T)])
    full = oracle.full_attn_select(qr, oracle.rope_rows(K, np.arange(T)), V, range(T), 0, 4, 3)
    for t in range(T):
        assert np.allclose(got[t], full[t].O, rtol=1e-12, atol=1e-12)
