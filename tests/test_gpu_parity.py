"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Sizes the oracle finishes in seconds that still span several tiles and a
ragged tail; edge cases (rows with fewer candidates than top-k, fewer keys
than the window, a single query, chunked prefill, invalid idx entries, the
bounded-wait timeout path)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from hs2_cases import (abs_dot, bf16_rule, check_select_rows, fp8_rule, gpu_decode_select, gpu_prefill_select,
                       gpu_sparse_decode, gpu_sparse_prefill)
from parity import TOL_BF16, TOL_FP8, check_block_row, check_idx_row, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hs2():
    import token_level_kv_b200 as m
    return m


# ---------------------------------------------------------------- bridging

@pytest.mark.parametrize("rows,D", [(333, 2048), (128, 512), (1, 64)])
def test_bridge_bf16(hs2, rows, D):
    c = synth.make_bridge_case(rows, D, 256, 1, seed=1)
    h, Wk, Wv = c.hidden.cuda(), c.Wk[0].cuda(), c.Wv[0].cuda()
    K = torch.empty(rows, 256, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    hs2.hs2_bridge_kv(h, Wk, Wv, K, V)
    assert hs2.hs2_device_status() == 0
    for got, W in ((K, c.Wk[0]), (V, c.Wv[0])):
        exact = oracle.bridge_rows(c.hidden, W)
        bad, err = bf16_rule(got.cpu(), exact, abs_dot(c.hidden, W))
        assert bad == 0, f"{bad} bf16 outputs off by more than the rounding rule (max err {err})"


@pytest.mark.parametrize("rows", [333, 1000])
def test_bridge_fp8(hs2, rows):
    c = synth.make_bridge_case(rows, 2048, 256, 1, seed=2)
    c.hidden[5] = 0          # an all-zero hidden row -> all-zero K/V row, scale 1
    h, Wk, Wv = c.hidden.cuda(), c.Wk[0].cuda(), c.Wv[0].cuda()
    K = torch.empty(rows, 256, dtype=torch.uint8, device="cuda")
    V = torch.empty_like(K)
    ks = torch.empty(rows, dtype=torch.float32, device="cuda")
    vs = torch.empty_like(ks)
    hs2.hs2_bridge_kv(h, Wk, Wv, K, V, ks, vs)
    assert hs2.hs2_device_status() == 0
    for codes, sc, W in ((K, ks, c.Wk[0]), (V, vs, c.Wv[0])):
        exact = oracle.bridge_rows(c.hidden, W)
        assert float(sc[5]) == 1.0 and int(codes[5].abs().sum()) == 0
        nz = np.abs(exact).max(1) > 0
        sbad, bad = fp8_rule(codes.cpu()[nz], sc.cpu()[nz], exact[nz], abs_dot(c.hidden, W)[nz])
        assert sbad == 0, f"{sbad} row scales off by more than the accumulation bound"
        assert bad == 0, f"{bad} FP8 codes off by more than the rounding rule"


def test_bridge_append_writes_one_fp8_row_per_sequence(hs2):
    """Decode-step bridging: each sequence's new hidden row is projected and its
    FP8 K/V row and scales written at pos[b]; every other cache byte is left
    as it was; an out-of-range pos is reported and skipped."""
    B, S, D, d = 6, 300, 2048, 256
    c = synth.make_bridge_case(B, D, d, 1, seed=15)
    c.hidden[3] = 0                       # all-zero row: codes 0, scale 1
    g = torch.Generator().manual_seed(0)
    Kc = torch.randint(0, 255, (B, S, d), dtype=torch.uint8, generator=g)
    Vc = torch.randint(0, 255, (B, S, d), dtype=torch.uint8, generator=g)
    ks = torch.rand(B, S, generator=g)
    vs = torch.rand(B, S, generator=g)
    pos = torch.tensor([0, 17, 299, 5, 100, 299], dtype=torch.int32)
    dev = [t.cuda() for t in (Kc, Vc, ks, vs)]
    hs2.hs2_bridge_append(c.hidden.cuda(), c.Wk[0].cuda(), c.Wv[0].cuda(), *dev, pos.cuda())
    assert hs2.hs2_device_status() == 0
    Kg, Vg, ksg, vsg = (t.cpu() for t in dev)
    rows = torch.arange(B)
    for got, before, sc, sc_before, W in ((Kg, Kc, ksg, ks, c.Wk[0]), (Vg, Vc, vsg, vs, c.Wv[0])):
        mask = torch.ones(B, S, dtype=torch.bool)
        mask[rows, pos.long()] = False
        assert torch.equal(got[mask], before[mask]) and torch.equal(sc[mask], sc_before[mask])
        codes, scales = got[rows, pos.long()], sc[rows, pos.long()]
        exact = oracle.bridge_rows(c.hidden, W)
        assert float(scales[3]) == 1.0 and int(codes[3].sum()) == 0
        nz = np.abs(exact).max(1) > 0
        sbad, bad = fp8_rule(codes[nz], scales[nz], exact[nz], abs_dot(c.hidden, W)[nz])
        assert sbad == 0 and bad == 0
    bad_pos = pos.clone()
    bad_pos[2] = S                        # one row past the cache
    hs2.hs2_bridge_append(c.hidden.cuda(), c.Wk[0].cuda(), c.Wv[0].cuda(), *dev, bad_pos.cuda())
    assert hs2.hs2_device_status() == 6   # HS2_ERR_DEVICE_CHECK, and nothing written for it
    assert torch.equal(dev[0][2].cpu(), Kg[2])


# ---------------------------------------------------------------- prefill select

def test_prefill_select_small_h8_d128(hs2):
    """1024 queries, 8 heads, d = 128, window 128 + top-256, 4 needles: all rows."""
    c = synth.CONFIGS[1]
    case = synth.make_prefill_case(c["T"], c["H"], c["d"], c["window"], c["topk"], n_sparse=1,
                                   n_needles=c["n_needles"], seed=0)
    O, idx = gpu_prefill_select(case)
    ref, worst, swaps = check_select_rows(case, O, idx, range(case.T))
    for p, i in case.needles:
        assert p in set(idx[i, case.window:].tolist())
    # sparse layer on the oracle's index set (identical inputs on both sides)
    oidx = np.stack([ref[t].idx for t in range(case.T)])
    Os = gpu_sparse_prefill(case.Q_sparse[0], case.K, case.V, oidx)
    sref = oracle.sparse_attn(case.Q_sparse[0], case.K, case.V, oidx, range(case.T))
    assert max(max_abs(Os[t].float().numpy(), sref[t]) for t in range(case.T)) <= TOL_BF16
    # end to end on the GPU's own index set where it equals the oracle's
    Os2 = gpu_sparse_prefill(case.Q_sparse[0], case.K, case.V, idx.numpy())
    same = [t for t in range(case.T) if np.array_equal(idx[t].numpy(), oidx[t])]
    assert len(same) >= case.T // 2
    assert max(max_abs(Os2[t].float().numpy(), sref[t]) for t in same) <= TOL_BF16


@pytest.mark.parametrize("T", [1500, 200, 1])
def test_prefill_select_h16_d256(hs2, T):
    """16 heads, d = 256, window 128 + top-1024: rows with fewer candidates
    than top-k, fewer keys than the window, a ragged last query tile."""
    case = synth.make_prefill_case(T, 16, 256, 128, 1024, n_sparse=1, n_needles=2 if T > 300 else 0,
                                   seed=4)
    O, idx = gpu_prefill_select(case)
    rows = range(T)
    check_select_rows(case, O, idx, rows)


def test_prefill_select_scaled_inputs_tie_margin(hs2):
    """N(0,1)/16 inputs: near-uniform attention, selection decided by tiny gaps."""
    case = synth.make_prefill_case(2600, 16, 256, 128, 1024, n_sparse=0, n_needles=8, scale=1 / 16, seed=5)
    O, idx = gpu_prefill_select(case)
    rows = list(range(1100, 1200)) + list(range(2500, 2600)) + [i for _, i in case.needles]
    _, _, swaps = check_select_rows(case, O, idx, rows)
    for p, i in case.needles:
        assert p in set(idx[i, case.window:].tolist())


def test_chunked_prefill_equals_one_call(hs2):
    """Query chunks over the causal prefix give the same rows, bit for bit."""
    case = synth.make_prefill_case(1800, 16, 256, 128, 1024, n_sparse=0, seed=6)
    O1, idx1 = gpu_prefill_select(case)
    Oa, idxa = gpu_prefill_select(case, q_start=0, Tq=904)
    Ob, idxb = gpu_prefill_select(case, q_start=904, Tq=896)
    assert torch.equal(torch.cat([idxa, idxb]), idx1)
    assert torch.equal(torch.cat([Oa, Ob]), O1)
    check_select_rows(case, Ob, idxb, [0, 1, 500, 895], q_start=904)


@pytest.mark.parametrize("T,H,d,W,B,k,scale", [(2600, 16, 256, 128, 64, 16, 1 / 16), (1500, 8, 128, 128, 32, 8, 1.0),
                                                (700, 16, 256, 64, 256, 4, 1.0), (900, 16, 128, 32, 16, 40, 1.0),
                                                (300, 16, 256, 128, 64, 16, 1.0)])
def test_prefill_block_selection(hs2, T, H, d, W, B, k, scale):
    """Block-level selection on the GPU against the oracle: whole blocks, the
    block set within the tie margin, the same full-attention output; rows with
    fewer candidate blocks than k (all taken), a partial boundary block, near
    uniform attention (scale 1/16) and several block sizes."""
    case = synth.make_prefill_case(T, H, d, W, k * B, n_sparse=0, scale=scale, seed=16)
    Q, K, V = case.Q.cuda(), case.K.cuda(), case.V.cuda()
    O = torch.empty(T, H, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(T, W + k * B, dtype=torch.int32, device="cuda")
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_BF16, 1, T, T, H, d, W, k))
    hs2.hs2_full_attn_select_blocks(Q, K, V, O, idx, ws, window=W, block=B, topk_blocks=k)
    assert hs2.hs2_device_status() == 0
    rows = sorted(set(list(range(0, T, 37)) + [W - 1, W, W + B - 1, W + B, W + k * B, T - 1]) & set(range(T)))
    ref = oracle.full_attn_select_blocks(case.Q, case.K, case.V, rows, 0, W, B, k)
    idx_c, O_c = idx.cpu().numpy(), O.float().cpu().numpy()
    for t in rows:
        r, b = ref[t]
        ok, _, msg = check_block_row(idx_c[t], b, W, B, k)
        assert ok, msg
        assert max_abs(O_c[t], r.O) <= TOL_BF16


def test_decode_block_selection_fp8(hs2):
    B, N, Bk, k = 3, 5000, 64, 16
    case = synth.make_decode_case(B, N, 16, 256, 128, k * Bk, n_sparse=0, seed=17)
    O = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(B, 128 + k * Bk, dtype=torch.int32, device="cuda")
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_FP8_E4M3, B, 1, N, 16, 256, 128, k))
    dev = [t.cuda() for t in (case.Q, case.Kc, case.Vc, case.ks, case.vs)]
    hs2.hs2_full_attn_select_blocks(dev[0], dev[1], dev[2], O, idx, ws, window=128, block=Bk, topk_blocks=k,
                                    k_scale=dev[3], v_scale=dev[4])
    assert hs2.hs2_device_status() == 0
    ref = oracle.decode_select(case.Q, case.Kc, case.Vc, case.ks, case.vs, range(B), N, 128, 1)
    for b in range(B):
        blk = oracle.block_select_row(ref[b].sigma, N - 1, 128, Bk, k)
        ok, _, msg = check_block_row(idx[b].cpu().numpy(), blk, 128, Bk, k)
        assert ok, msg
        assert max_abs(O[b].float().cpu().numpy(), ref[b].O) <= TOL_FP8


@pytest.mark.parametrize("T,H,d,W,q_start", [(1500, 16, 256, 128, 0), (1500, 8, 128, 64, 0), (900, 16, 256, 300, 700),
                                            (100, 16, 256, 128, 0), (2600, 16, 128, 1, 0)])
def test_swa_attn_partial_rope(hs2, T, H, d, W, q_start):
    """Self-decoder sliding-window attention with 64-dim partial RoPE against
    the oracle: windows of 1, 64, 128 and 300 keys, a query block starting at
    700 over the causal prefix, rows with fewer keys than the window."""
    kv = q_start + T
    case = synth.make_prefill_case(kv, H, d, W, 8, n_sparse=0, seed=20)
    Q = case.Q[q_start:kv].cuda().contiguous()
    O = torch.empty(T, H, d, dtype=torch.bfloat16, device="cuda")
    ws = hs2.workspace(hs2.hs2_swa_attn_prefill_workspace(T, kv, H, d))
    hs2.hs2_swa_attn_prefill(Q, case.K.cuda(), case.V.cuda(), O, ws, window=W, q_start=q_start)
    assert hs2.hs2_device_status() == 0
    rows = sorted(set(list(range(0, T, 29)) + [0, 1, W - 1, W, W + 1, T - 1]) & set(range(T)))
    ref = oracle.swa_attn(case.Q[q_start:kv], case.K, case.V, rows, q_start, W)
    Oc = O.float().cpu().numpy()
    assert max(max_abs(Oc[t], ref[t]) for t in rows) <= TOL_BF16


def test_swa_chunked_equals_one_call(hs2):
    T, H, d, W = 1800, 16, 256, 128
    case = synth.make_prefill_case(T, H, d, W, 8, n_sparse=0, seed=21)
    Q, K, V = case.Q.cuda(), case.K.cuda(), case.V.cuda()
    ws = hs2.workspace(hs2.hs2_swa_attn_prefill_workspace(T, T, H, d))
    O1 = torch.empty(T, H, d, dtype=torch.bfloat16, device="cuda")
    hs2.hs2_swa_attn_prefill(Q, K, V, O1, ws, window=W)
    O2 = torch.empty_like(O1)
    hs2.hs2_swa_attn_prefill(Q[:904].contiguous(), K, V, O2[:904], ws, window=W, kv_len=904)
    hs2.hs2_swa_attn_prefill(Q[904:].contiguous(), K, V, O2[904:], ws, window=W, q_start=904)
    assert hs2.hs2_device_status() == 0
    assert torch.equal(O1, O2)


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("B,N", [(3, 5000), (2, 1200), (1, 100), (2, 4097)])
def test_decode_select_fp8(hs2, B, N):
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=1, seed=7)
    O, idx = gpu_decode_select(case)
    ref = oracle.decode_select(case.Q, case.Kc, case.Vc, case.ks, case.vs, range(B), N, 128, 1024)
    for b in range(B):
        ok, _, msg = check_idx_row(idx[b].numpy(), ref[b], 128, 1024)
        assert ok, msg
        assert max_abs(O[b].float().numpy(), ref[b].O) <= TOL_FP8
    oidx = np.stack([ref[b].idx for b in range(B)])
    Os = gpu_sparse_decode(case, case.Q_sparse[0], oidx)
    sref = oracle.sparse_attn_decode(case.Q_sparse[0], case.Kc, case.Vc, case.ks, case.vs, oidx, range(B))
    for b in range(B):
        assert max_abs(Os[b].float().numpy(), sref[b]) <= TOL_FP8


@pytest.mark.parametrize("B,N", [(2, 140000), (1, 300000)])
def test_decode_select_split_topk(hs2, B, N):
    """Rows of more than 131072 candidates take the radix select over the whole
    GPU (chunks of 8192 candidates adding to three digit histograms, then
    a count and an ordered write): checked against the oracle."""
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=0, seed=18)
    O, idx = gpu_decode_select(case)
    ref = oracle.decode_select(case.Q, case.Kc, case.Vc, case.ks, case.vs, range(B), N, 128, 1024)
    for b in range(B):
        ok, _, msg = check_idx_row(idx[b].numpy(), ref[b], 128, 1024)
        assert ok, msg
        assert max_abs(O[b].float().numpy(), ref[b].O) <= TOL_FP8


def test_decode_split_topk_exact_ties_go_to_smaller_positions(hs2):
    """Every key identical: every candidate score is the same fp32 value, so the
    selection must be positions 0..1023 exactly, across the chunk boundaries."""
    B, N = 2, 300000
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=0, seed=19)
    case.Kc[:] = case.Kc[:, :1]
    case.ks[:] = case.ks[:, :1]
    O, idx = gpu_decode_select(case)
    for b in range(B):
        assert idx[b, 128:].tolist() == list(range(1024))
        assert idx[b, :128].tolist() == list(range(N - 128, N))


def test_decode_radix_ties_inside_the_cut(hs2):
    """Rows of 199,872 candidates (the radix select) with 300 strong keys and a
    run of identical keys at every 37th other position: the selection is the
    strong keys plus the first 724 tied keys in position order, a tie run that
    crosses chunk boundaries and is cut inside (the ties taken are fewer than
    the ties present); checked against the oracle exactly."""
    from hs2_cases import plant_tie_keys
    B, N, k = 2, 200000, 1024
    case = synth.make_decode_case(B, N, 16, 256, 128, k, n_sparse=0, seed=21)
    planted = plant_tie_keys(case)
    O, idx = gpu_decode_select(case)
    ref = oracle.decode_select(case.Q, case.Kc, case.Vc, case.ks, case.vs, range(B), N, 128, k)
    for b in range(B):
        strong, ties = planted[b]
        want = np.sort(np.concatenate([strong, ties[:k - len(strong)]]))
        assert np.array_equal(ref[b].idx[128:], want)                 # the oracle agrees with the construction
        assert np.array_equal(idx[b, 128:].numpy(), want)
        assert ties[k - len(strong) - 1] > 2 * 8192 and len(ties) > k - len(strong)   # across chunks, cut inside
        assert max_abs(O[b].float().numpy(), ref[b].O) <= TOL_FP8


def test_sparse_decode_many_sequences(hs2):
    """More sequences than SMs' worth of splits, kv_len below the row stride."""
    B, N = 70, 3000
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=1, seed=8)
    g = np.random.default_rng(0)
    idx = np.full((B, 1152), -1, dtype=np.int32)
    for b in range(B):
        n = int(g.integers(1, 1153))
        idx[b, :n] = np.sort(g.choice(2900, size=n, replace=False))
    O = gpu_sparse_decode(case, case.Q_sparse[0], idx, kv_len=2900)
    ref = oracle.sparse_attn_decode(case.Q_sparse[0], case.Kc, case.Vc, case.ks, case.vs, idx, range(B))
    assert max(max_abs(O[b].float().numpy(), ref[b]) for b in range(B)) <= TOL_FP8


@pytest.mark.parametrize("n_idx,H,d", [(1920, 16, 256), (1793, 16, 256), (1792, 16, 256), (1920, 8, 128),
                                       (1921, 16, 256), (2000, 16, 256), (1300, 8, 128), (5, 16, 256)])
def test_sparse_prefill_index_widths(hs2, n_idx, H, d):
    """Index rows at the tensor-core kernel's limit (15 tiles of 128 keys: 1920, and 1793,
    the first width that needs the 15th tile), one tile below it, just past it (1921 and
    2000: the warp-pair kernel), a ragged H = 8, d = 128 case and a tiny one, each with
    empty (-1) slots scattered through the row and repeated keys; sampled rows against the
    oracle."""
    T = 2200
    case = synth.make_prefill_case(T, H, d, 128, 64, n_sparse=1, seed=11)
    rng = np.random.default_rng(n_idx)
    idx = np.sort(rng.integers(0, T, size=(T, n_idx)), axis=1).astype(np.int32)
    idx[rng.random((T, n_idx)) < 0.05] = -1
    idx[:, 0] = np.arange(T)                  # every row keeps one real key
    O = gpu_sparse_prefill(case.Q_sparse[0], case.K, case.V, idx)
    rows = list(range(0, T, 173)) + [T - 1]
    ref = oracle.sparse_attn(case.Q_sparse[0], case.K, case.V, idx, rows)
    assert max(max_abs(O[t].float().numpy(), ref[t]) for t in rows) <= TOL_BF16


def test_rows_with_no_valid_entry_give_zero(hs2):
    """A row whose idx holds no valid entry selects nothing: its output is
    exactly zero and nothing is reported, on the prefill kernel and on both
    decode paths (a cluster per sequence at 70 sequences; split partials at 1)."""
    T, H, d = 300, 16, 256
    case = synth.make_prefill_case(T, H, d, 128, 64, n_sparse=1, seed=12)
    idx = np.full((T, 192), -1, dtype=np.int32)
    for t in range(T):
        idx[t, :min(t + 1, 192)] = np.arange(max(0, t - 191), t + 1)
    empty = [0, 7, 150, T - 1]
    idx[empty] = -1
    O = gpu_sparse_prefill(case.Q_sparse[0], case.K, case.V, idx)
    for t in empty:
        assert torch.count_nonzero(O[t]) == 0
    rows = [1, 8, 151, 298]
    ref = oracle.sparse_attn(case.Q_sparse[0], case.K, case.V, idx, rows)
    assert max(max_abs(O[t].float().numpy(), ref[t]) for t in rows) <= TOL_BF16
    for B in (70, 1, 3):
        dc = synth.make_decode_case(B, 2000, 16, 256, 128, 1024, n_sparse=1, seed=13)
        g = np.random.default_rng(B)
        didx = np.sort(g.integers(0, 2000, size=(B, 1152)), axis=1).astype(np.int32)
        gone = [0] if B == 1 else [0, B - 1]
        didx[gone] = -1
        Od = gpu_sparse_decode(dc, dc.Q_sparse[0], didx)
        for b in gone:
            assert torch.count_nonzero(Od[b]) == 0
        live = [b for b in range(B) if b not in gone][:4]
        if live:
            dref = oracle.sparse_attn_decode(dc.Q_sparse[0], dc.Kc, dc.Vc, dc.ks, dc.vs, didx, live)
            assert max(max_abs(Od[b].float().numpy(), dref[b]) for b in live) <= TOL_FP8


@pytest.mark.parametrize("B,N", [(3, 5000), (70, 1500)])
def test_decode_small_value_scales(hs2, B, N):
    """A cache whose V scales are 2^-16 of the usual ones: every output is 2^-16
    of the usual one.  The kernels hold p * v_scale in f16 against a per-row
    power-of-two reference, so the result is the unscaled run's times 2^-16,
    bit for bit, and the error relative to the output stays the unscaled one
    (no f16 underflow), for the full layer and the sparse layer."""
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=1, seed=14)
    O1, idx1 = gpu_decode_select(case)
    oidx = idx1.numpy()
    Os1 = gpu_sparse_decode(case, case.Q_sparse[0], oidx)
    small = synth.DecodeCase(case.B, case.N, case.H, case.d, case.window, case.topk, case.Q, case.Kc, case.Vc,
                             case.ks, case.vs * 2.0 ** -16, case.Q_sparse)
    O2, idx2 = gpu_decode_select(small)
    Os2 = gpu_sparse_decode(small, small.Q_sparse[0], oidx)
    assert torch.equal(idx1, idx2)
    assert torch.equal(O2.float(), O1.float() * 2.0 ** -16)
    assert torch.equal(Os2.float(), Os1.float() * 2.0 ** -16)
    seqs = [0, B - 1]
    ref = oracle.decode_select(small.Q, small.Kc, small.Vc, small.ks, small.vs, seqs, N, 128, 1024)
    sref = oracle.sparse_attn_decode(small.Q_sparse[0], small.Kc, small.Vc, small.ks, small.vs, oidx, seqs)
    for b in seqs:
        for got, want in ((O2[b], ref[b].O), (Os2[b], sref[b])):
            assert max_abs(got.float().numpy(), want) <= TOL_FP8 * 2.0 ** -16


# ---------------------------------------------------------------- checks and faults

def test_sparse_prefill_bad_index_is_reported_and_skipped(hs2):
    T, H, d = 40, 16, 128
    case = synth.make_prefill_case(T, H, d, 8, 8, n_sparse=1, seed=9)
    idx = np.full((T, 16), -1, dtype=np.int32)
    for t in range(T):
        idx[t, :t + 1 if t < 16 else 16] = np.arange(min(t + 1, 16))
    bad = idx.copy()
    bad[3, 1] = 10 ** 6                       # outside the KV
    O = torch.empty(T, H, d, dtype=torch.bfloat16, device="cuda")
    hs2.hs2_sparse_attn_prefill(case.Q_sparse[0].cuda(), case.K.cuda(), case.V.cuda(),
                                torch.from_numpy(bad).cuda(), O)
    assert hs2.hs2_device_status() == 6      # HS2_ERR_DEVICE_CHECK
    assert hs2.hs2_device_status() == 0      # the word is cleared once read
    skipped = idx.copy()
    skipped[3, 1] = -1
    ref = oracle.sparse_attn(case.Q_sparse[0], case.K, case.V, skipped, range(T))
    assert max(max_abs(O[t].float().cpu().numpy(), ref[t]) for t in range(T)) <= TOL_BF16


def test_argument_errors_do_not_launch(hs2):
    K = torch.empty(10, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hs2.Hs2Error) as e:
        hs2.hs2_bridge_kv(torch.empty(10, 100, dtype=torch.bfloat16, device="cuda"),
                          torch.empty(256, 100, dtype=torch.bfloat16, device="cuda"),
                          torch.empty(256, 100, dtype=torch.bfloat16, device="cuda"), K, K)
    assert e.value.status == 1
    Q = torch.empty(4, 16, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hs2.Hs2Error) as e:
        hs2.hs2_full_attn_select(Q, K, K, Q, torch.empty(4, 1152, dtype=torch.int32, device="cuda"),
                                 torch.empty(64, dtype=torch.uint8, device="cuda"), window=128, topk=1024)
    assert e.value.status == 3               # workspace too small
    with pytest.raises(hs2.Hs2Error) as e:
        hs2.hs2_full_attn_select(torch.empty(4, 12, 256, dtype=torch.bfloat16, device="cuda"), K, K, Q,
                                 torch.empty(4, 1152, dtype=torch.int32, device="cuda"),
                                 torch.empty(1 << 20, dtype=torch.uint8, device="cuda"), window=128, topk=1024)
    assert e.value.status == 2               # 12 heads: unsupported
    assert hs2.hs2_device_status() == 0


def test_bounded_wait_gives_up_and_context_survives(hs2):
    """With a wait limit of one try the tensor-core kernel's waits give up: the
    call reports HS2_ERR_TIMEOUT through the status word, the CTAs drain their
    own copies and MMAs, and the next call with the default limit is exact."""
    c = synth.make_bridge_case(4096, 2048, 256, 1, seed=3)
    h, Wk, Wv = c.hidden.cuda(), c.Wk[0].cuda(), c.Wv[0].cuda()
    K = torch.empty(4096, 256, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    hs2.hs2_set_spin_limit(1)
    try:
        hs2.hs2_bridge_kv(h, Wk, Wv, K, V)
        st = hs2.hs2_device_status()
    finally:
        hs2.hs2_set_spin_limit(0)
    assert st == 5                           # HS2_ERR_TIMEOUT
    hs2.hs2_bridge_kv(h, Wk, Wv, K, V)
    assert hs2.hs2_device_status() == 0
    bad, _ = bf16_rule(K[:300].cpu(), oracle.bridge_rows(c.hidden[:300], c.Wk[0]),
                       abs_dot(c.hidden[:300], c.Wk[0]))
    assert bad == 0


def test_fp8_widening_is_exact_for_every_code(hs2):
    """One selected key: its probability is 1 and O = v_scale * E4M3(V row), so
    the bf16 output reproduces all 254 finite codes (subnormals included)."""
    d = 256
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    codes[0x7F] = 0
    codes[0xFF] = 0                            # the two NaN codes are not stored
    Vc = torch.zeros(1, 16, d, dtype=torch.uint8)
    Vc[0, 3] = codes
    Kc = torch.randint(0, 0x7E, (1, 16, d), dtype=torch.uint8)
    ks = torch.ones(1, 16)
    vs = torch.ones(1, 16)
    Q = synth.normal_bf16(0, 1, (1, 16, d))
    idx = torch.full((1, 16), -1, dtype=torch.int32)
    idx[0, 0] = 3
    O = torch.empty(1, 16, d, dtype=torch.bfloat16, device="cuda")
    ws = hs2.workspace(hs2.hs2_sparse_attn_decode_workspace(1, 16, 16, d))
    hs2.hs2_sparse_attn_decode(Q.cuda(), Kc.cuda(), Vc.cuda(), ks.cuda(), vs.cuda(), idx.cuda(), O, ws)
    assert hs2.hs2_device_status() == 0
    want = torch.from_numpy(oracle.e4m3_decode(codes.numpy()))
    for h in range(16):
        assert torch.equal(O[0, h].double().cpu(), want)
