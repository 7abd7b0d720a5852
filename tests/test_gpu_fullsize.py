"""Full-size workloads, in the launch configuration bench.py times, checked on
sampled rows / sequences that the fp64 oracle computes one by one.

* prefill T = 32768, 16 heads, d = 256, N(0,1)/16 + 64 needles, 3 sparse layers
* decode over an FP8 cache, 64 sequences x 131072 tokens, 3 sparse layers
* chunked prefill T = 262144 (8192-query chunks), Zipf key norms, 2 sparse layers
* bridged 1M decode: bridging of 4 x 2^20 hidden rows into 2 layers' FP8
  caches, then decode of 4 sequences x 2^20 tokens in both layers (full
  attention + selection and 3 sparse layers each) over those bridged caches
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from hs2_cases import abs_dot, fp8_rule
from parity import TOL_BF16, TOL_FP8, check_idx_row, max_abs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def hs2():
    import token_level_kv_b200 as m
    return m


def _rows(T, n, seed, extra=()):
    g = np.random.default_rng(seed)
    rows = set(int(x) for x in g.integers(0, T, size=n))
    rows.update(r for r in extra if 0 <= r < T)
    return sorted(rows)


def _select_and_sparse(hs2, case, rows, q_start=0, Tq=None):
    """One full-attention+select call over queries [q_start, q_start+Tq) and the
    sparse layers; oracle rows compared under the parity rules."""
    T, H, d, W, k = case.T, case.H, case.d, case.window, case.topk
    Tq = T - q_start if Tq is None else Tq
    kv = q_start + Tq
    dev = case.Q.device
    Qb = case.Q[q_start:kv]
    O = torch.empty(Tq, H, d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(Tq, W + k, dtype=torch.int32, device=dev)
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_BF16, 1, Tq, kv, H, d, W, k), dev)
    hs2.hs2_full_attn_select(Qb, case.K[:kv], case.V[:kv], O, idx, ws, window=W, topk=k, q_start=q_start)
    assert hs2.hs2_device_status() == 0
    del ws
    Kc, Vc = oracle.f64(case.K[:kv].cpu()), oracle.f64(case.V[:kv].cpu())
    Qrows = Qb[rows].cpu()
    ref = oracle.full_attn_select(Qrows, Kc, Vc, [], 0, W, k)  # warm import
    worst, swaps = 0.0, 0
    oidx = idx.clone()
    idx_cpu = idx[rows].cpu().numpy()
    O_cpu = O[rows].float().cpu().numpy()
    refs = {}
    for n, t in enumerate(rows):
        r = oracle.select_row(oracle.f64(Qrows[n]), Kc, Vc, q_start + t, W, k, 1.0 / math.sqrt(d))
        refs[t] = r
        ok, sw, msg = check_idx_row(idx_cpu[n], r, W, k)
        assert ok, msg
        swaps += sw
        worst = max(worst, max_abs(O_cpu[n], r.O))
        oidx[t] = torch.from_numpy(r.idx).to(dev)
    assert worst <= TOL_BF16, f"full-attention output error {worst}"
    # sparse layers at full size, fed the oracle's index rows where sampled
    for l, Qs in enumerate(case.Q_sparse):
        Os = torch.empty(Tq, H, d, dtype=torch.bfloat16, device=dev)
        hs2.hs2_sparse_attn_prefill(Qs[q_start:kv], case.K[:kv], case.V[:kv], oidx, Os)
        assert hs2.hs2_device_status() == 0
        got = Os[rows].float().cpu().numpy()
        Qsr = Qs[q_start:kv][rows].cpu()
        for n, t in enumerate(rows):
            s = oracle.sparse_attn_row(oracle.f64(Qsr[n]), Kc, Vc, refs[t].idx, 1.0 / math.sqrt(d))
            assert max_abs(got[n], s) <= TOL_BF16
    return swaps


def test_prefill_32k_paper_shape(hs2):
    c = synth.CONFIGS[2]
    case = synth.make_prefill_case(c["T"], c["H"], c["d"], c["window"], c["topk"], c["n_sparse"],
                                   n_needles=c["n_needles"], scale=c["scale"], seed=0, device="cuda")
    T = c["T"]
    rows = _rows(T, 192, 1, extra=[0, 127, 128, 383, 1151, 1152, T - 1] + [i for _, i in case.needles])
    _select_and_sparse(hs2, case, rows)


def test_prefill_256k_chunked_zipf(hs2):
    c = synth.CONFIGS[4]
    case = synth.make_prefill_case(c["T"], c["H"], c["d"], c["window"], c["topk"], c["n_sparse"],
                                   zipf=True, scale=1.0, seed=0, device="cuda")
    ch = c["chunk"]
    # the first chunk (short rows, rows below the window) and the last (longest rows)
    for ci in (0, c["T"] // ch - 1):
        rows = _rows(ch, 24, 10 + ci, extra=[0, ch - 1] + ([127, 128, 1151, 1152] if ci == 0 else []))
        _select_and_sparse(hs2, case, rows, q_start=ci * ch, Tq=ch)


def _decode_layer(hs2, Q, Q_sparse, Kc, Vc, ks, vs, B, N, H, d, W, k, seqs, cpu=None):
    """Full layer (select) + its sparse layers over one FP8 cache, on the GPU,
    checked against the oracle on the sequences ``seqs``; the sparse layers are
    fed the oracle's index rows on those sequences (identical inputs)."""
    O = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(B, W + k, dtype=torch.int32, device="cuda")
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_FP8_E4M3, B, 1, N, H, d, W, k))
    hs2.hs2_full_attn_select(Q, Kc, Vc, O, idx, ws, window=W, topk=k, k_scale=ks, v_scale=vs)
    assert hs2.hs2_device_status() == 0
    del ws
    oidx = idx.clone()
    cpu = cpu or [t.cpu() for t in (Kc, Vc, ks, vs)]
    Qc = Q.cpu()
    for b in seqs:
        r = oracle.decode_select(Qc, *cpu, [b], N, W, k)[b]
        ok, _, msg = check_idx_row(idx[b].cpu().numpy(), r, W, k)
        assert ok, msg
        assert max_abs(O[b].float().cpu().numpy(), r.O) <= TOL_FP8
        oidx[b] = torch.from_numpy(r.idx).cuda()
    wss = hs2.workspace(hs2.hs2_sparse_attn_decode_workspace(B, W + k, H, d))
    for Qs in Q_sparse:
        Os = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
        hs2.hs2_sparse_attn_decode(Qs, Kc, Vc, ks, vs, oidx, Os, wss)
        assert hs2.hs2_device_status() == 0
        sref = oracle.sparse_attn_decode(Qs.cpu(), *cpu, oidx.cpu(), seqs)
        for b in seqs:
            assert max_abs(Os[b].float().cpu().numpy(), sref[b]) <= TOL_FP8


def _decode_full(hs2, case, seqs):
    _decode_layer(hs2, case.Q, case.Q_sparse, case.Kc, case.Vc, case.ks, case.vs, case.B, case.N, case.H,
                  case.d, case.window, case.topk, seqs)


def test_decode_64x128k_fp8(hs2):
    c = synth.CONFIGS[3]
    case = synth.make_decode_case(c["B"], c["N"], c["H"], c["d"], c["window"], c["topk"], c["n_sparse"],
                                  seed=0, device="cuda")
    _decode_full(hs2, case, range(c["B"]))


def test_bridged_decode_1m(hs2):
    """Bridging of every token of the 4 sequences into the 2 cross-decoder
    layers' FP8 caches (sampled rows against the oracle), then the decode step
    of BOTH layers -- full attention + selection and 3 sparse layers each --
    over those GPU-bridged caches, all 4 sequences against the oracle."""
    c = synth.CONFIGS[5]
    B, N, D, d, H, W, k = c["B"], c["N"], c["D"], c["d"], c["H"], c["window"], c["topk"]
    bc = synth.make_bridge_case(B * N, D, d, c["n_layers"], seed=0, device="cuda")
    rows = _rows(B * N, 2048, 3, extra=[0, B * N - 1, N - 1, N])
    caches = []
    for l in range(c["n_layers"]):
        K = torch.empty(B * N, d, dtype=torch.uint8, device="cuda")
        V = torch.empty_like(K)
        ks = torch.empty(B * N, dtype=torch.float32, device="cuda")
        vs = torch.empty_like(ks)
        hs2.hs2_bridge_kv(bc.hidden, bc.Wk[l], bc.Wv[l], K, V, ks, vs)
        assert hs2.hs2_device_status() == 0
        hr = bc.hidden[rows].cpu()
        for codes, sc, Wm in ((K, ks, bc.Wk[l]), (V, vs, bc.Wv[l])):
            Wc = Wm.cpu()
            exact = oracle.bridge_rows(hr, Wc)
            sbad, bad = fp8_rule(codes[rows].cpu(), sc[rows].cpu(), exact, abs_dot(hr, Wc))
            assert sbad == 0 and bad == 0
        caches.append((K.view(B, N, d), V.view(B, N, d), ks.view(B, N), vs.view(B, N)))
    del bc
    torch.cuda.empty_cache()
    queries = synth.bridged_decode_queries(B, H, d, c["n_layers"], c["n_sparse"], seed=0, device="cuda")
    for (Kc, Vc, ks, vs), (Q, Qs) in zip(caches, queries):
        _decode_layer(hs2, Q, Qs, Kc, Vc, ks, vs, B, N, H, d, W, k, range(B))
