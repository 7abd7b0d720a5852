"""Helpers shared by the GPU parity tests: run the CUDA path through the
binding, run the oracle on the same inputs, compare under the parity rules."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from parity import TOL_BF16, TOL_FP8, check_idx_row, max_abs


def gpu_prefill_select(case, q_start=0, Tq=None, kv_len=None):
    import token_level_kv_b200 as hs2
    Tq = case.T - q_start if Tq is None else Tq
    kv_len = q_start + Tq if kv_len is None else kv_len
    Q = case.Q[q_start:q_start + Tq].cuda().contiguous()
    K = case.K[:kv_len].cuda().contiguous()
    V = case.V[:kv_len].cuda().contiguous()
    H, d = case.H, case.d
    O = torch.empty(Tq, H, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(Tq, case.n_idx, dtype=torch.int32, device="cuda")
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_BF16, 1, Tq, kv_len, H, d,
                                                          case.window, case.topk))
    hs2.hs2_full_attn_select(Q, K, V, O, idx, ws, window=case.window, topk=case.topk, q_start=q_start,
                             kv_len=kv_len)
    st = hs2.hs2_device_status()
    assert st == 0, f"device status {hs2.STATUS.get(st)}"
    return O.cpu(), idx.cpu()


def check_select_rows(case, O, idx, rows, q_start=0, kv_len=None, tol=TOL_BF16, Ksrc=None, Vsrc=None):
    """Oracle on the given rows (indices into this call's query block)."""
    kv_len = q_start + O.shape[0] if kv_len is None else kv_len
    K = case.K[:kv_len] if Ksrc is None else Ksrc
    V = case.V[:kv_len] if Vsrc is None else Vsrc
    Qb = case.Q[q_start:q_start + O.shape[0]]
    ref = oracle.full_attn_select(Qb, K, V, rows, q_start, case.window, case.topk)
    worst, swaps = 0.0, 0
    for t in rows:
        r = ref[t]
        ok, n_sw, msg = check_idx_row(idx[t].numpy(), r, case.window, case.topk)
        assert ok, msg
        swaps += n_sw
        worst = max(worst, max_abs(O[t].float().numpy(), r.O))
    assert worst <= tol, f"full-attention output max-abs error {worst}"
    return ref, worst, swaps


def gpu_sparse_prefill(Qs, K, V, idx):
    import token_level_kv_b200 as hs2
    Tq, H, d = Qs.shape
    O = torch.empty(Tq, H, d, dtype=torch.bfloat16, device="cuda")
    hs2.hs2_sparse_attn_prefill(Qs.cuda().contiguous(), K.cuda().contiguous(), V.cuda().contiguous(),
                                torch.as_tensor(idx).cuda().contiguous(), O)
    st = hs2.hs2_device_status()
    assert st == 0, f"device status {hs2.STATUS.get(st)}"
    return O.cpu()


def gpu_decode_select(case, kv_len=None):
    import token_level_kv_b200 as hs2
    B, H, d = case.Q.shape
    N = case.N if kv_len is None else kv_len
    O = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(B, case.n_idx, dtype=torch.int32, device="cuda")
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_FP8_E4M3, B, 1, N, H, d, case.window,
                                                          case.topk))
    dev = [t.cuda().contiguous() for t in (case.Q, case.Kc, case.Vc, case.ks, case.vs)]
    hs2.hs2_full_attn_select(dev[0], dev[1], dev[2], O, idx, ws, window=case.window, topk=case.topk,
                             kv_len=N, k_scale=dev[3], v_scale=dev[4])
    st = hs2.hs2_device_status()
    assert st == 0, f"device status {hs2.STATUS.get(st)}"
    return O.cpu(), idx.cpu()


def gpu_sparse_decode(case, Qs, idx, kv_len=None):
    import token_level_kv_b200 as hs2
    B, H, d = Qs.shape
    N = case.N if kv_len is None else kv_len
    O = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    ws = hs2.workspace(hs2.hs2_sparse_attn_decode_workspace(B, idx.shape[-1], H, d))
    hs2.hs2_sparse_attn_decode(Qs.cuda().contiguous(), case.Kc.cuda(), case.Vc.cuda(), case.ks.cuda(),
                               case.vs.cuda(), torch.as_tensor(idx).cuda().contiguous(), O, ws, kv_len=N)
    st = hs2.hs2_device_status()
    assert st == 0, f"device status {hs2.STATUS.get(st)}"
    return O.cpu()


# fp32 accumulation on the tensor cores: the K-long dot product is summed as
# K/16 fp32 additions of 16-product partial sums, each rounded to fp32, so the
# fp32 value f obeys |f - exact| <= (K/16) * 2^-24 * sum_e |h_e w_e|, bounded
# here by 2^-17 * sum_e |h_e w_e| for K <= 2048.  The stored value is then one
# round-to-nearest-even of f.
ACC_REL = 2.0 ** -17


def abs_dot(hidden, W):
    return np.abs(oracle.f64(hidden)) @ np.abs(oracle.f64(W)).T


def bf16_rule(gpu, exact, sabs):
    """Count GPU bf16 values farther from the fp64 value than half a bf16 ulp
    plus the fp32 accumulation bound."""
    g = gpu.double().numpy()
    e = np.asarray(exact, dtype=np.float64)
    dlt = ACC_REL * sabs
    ulp = np.ldexp(1.0, np.frexp(np.abs(e) + dlt)[1] - 8)  # bf16: 8 significant bits
    err = np.abs(g - e)
    bad = err > 0.5 * ulp + dlt
    return int(bad.sum()), float(err.max())


def fp8_rule(codes, scales, exact, sabs):
    """FP8 rows: each scale is amax/448 up to the accumulation bound of the amax
    element; each code is within half an E4M3 ulp of x/scale plus the bound."""
    e = np.asarray(exact, dtype=np.float64)
    dlt = ACC_REL * sabs
    amax = np.abs(e).max(axis=1)
    sref = np.where(amax > 0, amax / 448.0, 1.0)
    s = scales.double().numpy()
    stol = dlt.max(axis=1) / np.maximum(amax, 1e-300) + 2.0 ** -23
    sbad = int((np.abs(s - sref) / sref > stol).sum())
    y = e / s[:, None]                                      # against the stored scale
    yg = oracle.e4m3_decode(codes.numpy())
    a = np.abs(y) + dlt / s[:, None]
    ex = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    ulp = np.ldexp(1.0, (ex - 3).astype(np.int64))        # 3 mantissa bits; subnormal ulp 2^-9
    # x/scale is one fp32 division (2^-24 relative) of the accumulated value
    bad = np.abs(yg - np.clip(y, -448, 448)) > 0.5 * ulp + dlt / s[:, None] + 2.0 ** -22 * np.abs(y)
    return sbad, int(bad.sum())


def plant_tie_keys(case, n_strong: int = 300, tie_every: int = 37, seed: int = 5):
    """Decode case with a planted structure around the k-th score: per
    sequence, n_strong keys (random candidate positions) far above every
    random key, and one identical key at every tie_every-th other candidate
    position, between the strong keys and the random ones.  The identical keys
    tie exactly (same codes, same scale), so the selection takes all strong
    keys and then the tied keys in position order, and the cut falls inside
    the run of ties.  Returns {b: (strong positions, tie positions)}."""
    import numpy as np
    B, N, d = case.B, case.N, case.d
    g = np.random.default_rng(seed)
    n_cand = N - case.window
    out = {}
    for b in range(B):
        qbar = case.Q[b].float().mean(dim=0)
        u = qbar / qbar.norm()
        strong = np.sort(g.choice(n_cand, n_strong, replace=False))
        is_strong = np.zeros(n_cand, dtype=bool)
        is_strong[strong] = True
        ties = np.array([j for j in range(0, n_cand, tie_every) if not is_strong[j]], dtype=np.int64)
        for pos, c in ((strong, 64.0), (ties, 40.0)):
            v = (c * u).to(torch.bfloat16).float()
            sc = v.abs().max() / 448.0
            code = (v / sc).to(torch.float8_e4m3fn).view(torch.uint8)
            idx = torch.as_tensor(pos)
            case.Kc[b, idx] = code
            case.ks[b, idx] = sc
        out[b] = (strong, ties)
    return out
