"""fp64 CPU oracle for the HySparse2 KV Reuse hot path -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may
import this package.  It shares no code with the CUDA library and never
imports it; both sides only share the seeded input generator ``synth``.

Everything here is the plain definition of what the method computes, written
row by row in float64 with numpy (a matmul, an exp, a sort are the only library
steps).  Sources, by page and passage:

* "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing" (agihunt.info
  summary), paragraph on inner-level KV Reuse: the full-attention layer scores
  tokens one by one; the 128 most recent tokens are always put in the sparse
  selection and 1024 high-scoring out-of-window tokens are added; the sparse
  layers read the same full-attention KV.
* same page, next paragraph: MQA (one KV head), NoPE on full and sparse layers,
  the full layer is an oracle selector using exact attention scores.
* same page, the outer-level KV Bridging paragraph: a cross-decoder full
  layer's K/V are the source hidden state re-projected by that layer's own
  projections.
* same page, results table header "KV @1M (FP8)": the KV cache is stored FP8.
* 10100.com article, "evolution two": the selection adds *at most* 1024 tokens.

Readings where the pages are silent (the same readings the CUDA path uses):
head aggregation = sum over the query heads of the softmax probabilities;
window = positions [p-W+1, p] (it includes the query itself); candidates =
[0, p-W]; softmax scale 1/sqrt(d); ties in the score broken by smaller
position; FP8 = OCP E4M3FN, round-to-nearest-even, saturating at +-448, one
fp32 scale per token row = amax/448 (1 for an all-zero row).

Parity unpinned (no page fixes it; pinned only to the stated reading): the
head aggregation rule, the softmax scale and the tie order.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

import numpy as np

E4M3_MAX = 448.0


def f64(x) -> np.ndarray:
    """Any array (numpy, or a CPU torch tensor of any float dtype) as float64."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def u8(x) -> np.ndarray:
    if hasattr(x, "detach"):
        return x.detach().cpu().numpy().astype(np.uint8, copy=False)
    return np.asarray(x, dtype=np.uint8)


# ---------------------------------------------------------------------------
# FP8 E4M3FN (storage format of the KV cache)
# ---------------------------------------------------------------------------

def e4m3_value(code: int) -> float:
    """Value of one E4M3FN code: 1 sign, 4 exponent (bias 7), 3 mantissa bits;
    exponent field 0 is subnormal (2^-6 * m/8); code 0x7F/0xFF is NaN; no inf."""
    s = (code >> 7) & 1
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -v if s else v


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
# non-negative finite codes 0x00..0x7E in increasing value order
_POS_VALUES = E4M3_TABLE[:0x7F]


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Nearest E4M3FN code, ties to the even code, |x| >= 448 saturates to 448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    sign = np.signbit(x).astype(np.uint8) << 7
    hi = np.searchsorted(_POS_VALUES, a, side="left")          # first value >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    dlo = a - _POS_VALUES[lo]
    dhi = _POS_VALUES[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a >= E4M3_MAX, 0x7E, code).astype(np.uint8)
    code = np.where(np.isnan(x), 0x7F, code | sign).astype(np.uint8)
    return code


def quantize_rows_e4m3(X: np.ndarray):
    """Per-row FP8 storage: scale = amax/448 (1 if amax == 0), code = E4M3(x/scale).

    Returns (codes uint8 [R,d], scales float64 [R], pre-rounding values x/scale).
    """
    X = f64(X)
    amax = np.abs(X).max(axis=1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    y = X / scale[:, None]
    return e4m3_encode(y), scale, y


# ---------------------------------------------------------------------------
# KV Bridging
# ---------------------------------------------------------------------------

def bridge_rows(hidden: np.ndarray, W: np.ndarray) -> np.ndarray:
    """K_r = sum_c hidden[r,c] * W[:,c]  (W in [out, in] layout), fp64."""
    return f64(hidden) @ f64(W).T


# ---------------------------------------------------------------------------
# Full attention as the oracle selector, and the index set
# ---------------------------------------------------------------------------

@dataclass
class SelectRow:
    p: int                    # absolute position of the query
    O: np.ndarray             # [H, d] attention output (unrounded)
    m: np.ndarray             # [H] row max of the logits
    l: np.ndarray             # [H] sum of exp(s - m)
    sigma: np.ndarray         # [p+1] head-summed probabilities
    idx: np.ndarray           # [window + topk] int32
    tau: Optional[float]      # k-th largest sigma among candidates (None: all taken)
    n_sel: int


def window_slots(p: int, window: int) -> np.ndarray:
    """Forced recent window: slot w holds position p-window+1+w, -1 if negative."""
    pos = np.arange(p - window + 1, p + 1, dtype=np.int64)
    return np.where(pos >= 0, pos, -1).astype(np.int32)


def topk_positions(sigma_c: np.ndarray, k: int) -> np.ndarray:
    """The k candidates with the largest score, ties to the smaller position,
    returned in ascending position order (all of them if there are <= k)."""
    n = sigma_c.shape[0]
    if n <= k:
        return np.arange(n, dtype=np.int64)
    order = np.lexsort((np.arange(n), -sigma_c))   # by -sigma, then position
    return np.sort(order[:k])


def select_row(q: np.ndarray, K: np.ndarray, V: np.ndarray, p: int, window: int,
               topk: int, scale: float) -> SelectRow:
    """One query row of the full-attention layer (MQA, NoPE) and its index set.

    q: [H, d] fp64; K, V: [>= p+1, d] fp64 (the single KV head).
    """
    s = (q @ K[:p + 1].T) * scale                    # [H, p+1] logits
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    l = e.sum(axis=1)
    P = e / l[:, None]                               # exact softmax probabilities
    O = P @ V[:p + 1]                                # [H, d]
    sigma = P.sum(axis=0)                            # head-summed score per key
    n_cand = max(0, p - window + 1)                  # candidates 0 .. p-window
    sel = topk_positions(sigma[:n_cand], topk)
    tau = None
    if n_cand > topk:
        tau = float(np.sort(sigma[:n_cand])[-topk])
    idx = np.full(window + topk, -1, dtype=np.int32)
    idx[:window] = window_slots(p, window)
    idx[window:window + sel.shape[0]] = sel
    return SelectRow(p, O, m, l, sigma, idx, tau, int(sel.shape[0]))


@dataclass
class BlockSelectRow:
    p: int
    sigma: np.ndarray         # [p+1] head-summed probabilities
    block_score: np.ndarray   # [n_blocks] sum of sigma over each block's candidates
    blocks: np.ndarray        # selected block numbers, ascending
    idx: np.ndarray           # [window + topk_blocks * block] int32
    tau: Optional[float]      # k-th largest block score (None: all blocks taken)


def block_select_row(sigma: np.ndarray, p: int, window: int, block: int,
                     topk_blocks: int) -> BlockSelectRow:
    """Block-level selection (the ablation's alternative to token level).

    The pages compare token-level selection with block-level selection of
    64-token blocks at the same 1024-token budget (agihunt.info summary,
    ablation paragraph; 10100.com article, "evolution one": blocks of 64 or
    128 tokens).  Readings: blocks are aligned, block c = positions
    [c*block, (c+1)*block); a block's score is the sum of sigma over its
    out-of-window candidates (positions <= p - window), so the boundary block
    counts only those; the topk_blocks blocks with the largest score are taken
    (ties to the smaller block number, all of them if there are fewer), and the
    index row is the forced window, then every candidate position of the
    selected blocks ascending, then -1.
    """
    n_cand = max(0, p - window + 1)
    nb = (n_cand + block - 1) // block
    score = np.zeros(nb, dtype=np.float64)
    for c in range(nb):
        score[c] = sigma[c * block:min(n_cand, (c + 1) * block)].sum()
    chosen = topk_positions(score, topk_blocks)            # same rule as tokens
    tau = None
    if nb > topk_blocks:
        tau = float(np.sort(score)[-topk_blocks])
    idx = np.full(window + topk_blocks * block, -1, dtype=np.int32)
    idx[:window] = window_slots(p, window)
    pos = [j for c in chosen for j in range(c * block, min(n_cand, (c + 1) * block))]
    idx[window:window + len(pos)] = pos
    return BlockSelectRow(p, sigma, score, np.asarray(chosen, dtype=np.int64), idx, tau)


def full_attn_select_blocks(Q: np.ndarray, K: np.ndarray, V: np.ndarray, rows: Sequence[int],
                            q_start: int, window: int, block: int, topk_blocks: int,
                            scale: Optional[float] = None):
    """The full layer with block-level selection: per row the token-level
    SelectRow (its O, m, l, sigma; the token index set is not used) and the
    BlockSelectRow built from the same sigma."""
    d = Q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    K = f64(K)
    V = f64(V)
    out = {}
    for t in rows:
        r = select_row(f64(Q[t]), K, V, q_start + t, window, 1, scale)
        out[t] = (r, block_select_row(r.sigma, q_start + t, window, block, topk_blocks))
    return out


def full_attn_select(Q: np.ndarray, K: np.ndarray, V: np.ndarray, rows: Sequence[int],
                     q_start: int, window: int, topk: int,
                     scale: Optional[float] = None) -> Dict[int, SelectRow]:
    """Prefill: query t sits at absolute position q_start + t and sees keys <= it.

    Q: [Tq, H, d]; K, V: [kv_len, d] -- any float dtype, read as fp64.
    """
    d = Q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    K = f64(K)
    V = f64(V)
    out = {}
    for t in rows:
        q = f64(Q[t])
        out[t] = select_row(q, K, V, q_start + t, window, topk, scale)
    return out


def sparse_attn_row(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx_row: np.ndarray,
                    scale: float) -> np.ndarray:
    """Sparse layer: softmax attention of its own q over the selected keys only.

    An entry that appears twice in the row is attended twice (each slot is one
    key of the softmax).  A row with no valid entry selects nothing; its output
    is taken as zero (the empty sum), the library's stated convention."""
    S = idx_row[idx_row >= 0].astype(np.int64)
    if S.shape[0] == 0:
        return np.zeros((q.shape[0], V.shape[1]), dtype=np.float64)
    s = (q @ K[S].T) * scale                         # [H, |S|]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    P = e / e.sum(axis=1, keepdims=True)
    return P @ V[S]


def sparse_attn(Qs: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray,
                rows: Sequence[int], scale: Optional[float] = None) -> Dict[int, np.ndarray]:
    d = Qs.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    K = f64(K)
    V = f64(V)
    idx = idx.cpu().numpy() if hasattr(idx, "cpu") else np.asarray(idx)
    return {t: sparse_attn_row(f64(Qs[t]), K, V, idx[t], scale) for t in rows}


# ---------------------------------------------------------------------------
# Self-decoder sliding-window attention with partial RoPE
# ---------------------------------------------------------------------------

def rope_rows(X: np.ndarray, positions: np.ndarray, rope_dims: int = 64,
              base: float = 10000.0) -> np.ndarray:
    """Rotary position embedding on the first rope_dims dims of every row
    (agihunt.info summary: the SWA layers use 64-dim partial RoPE; full and
    sparse layers use NoPE).  Readings, the pages fixing none of them: pairs
    are (i, i + rope_dims/2) for i < rope_dims/2 (rotate-half), the angle of
    pair i at position p is p * base^(-2i/rope_dims) with base 10000, and the
    remaining dims pass through.

    X: [..., rows, d] (any leading dims), positions: [rows] absolute positions.
    """
    X = f64(X)
    half = rope_dims // 2
    inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / rope_dims)   # [half]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]    # [rows, half]
    shape = [1] * (X.ndim - 2) + [ang.shape[0], half]
    c = np.cos(ang).reshape(shape)
    sn = np.sin(ang).reshape(shape)
    out = X.copy()
    x1 = X[..., :half]
    x2 = X[..., half:rope_dims]
    out[..., :half] = x1 * c - x2 * sn
    out[..., half:rope_dims] = x1 * sn + x2 * c
    return out


def swa_attn(Q: np.ndarray, K: np.ndarray, V: np.ndarray, rows: Sequence[int], q_start: int,
             window: int, rope_dims: int = 64, base: float = 10000.0,
             scale: Optional[float] = None) -> Dict[int, np.ndarray]:
    """Sliding-window causal attention of the self-decoder (agihunt.info summary,
    backbone paragraph: each query attends only to the most recent tokens), MQA
    with one KV head, RoPE on q and k: query t at position p = q_start + t sees
    keys [max(0, p - window + 1), p].

    Q: [Tq, H, d]; K, V: [kv_len, d].  Returns {t: O [H, d]} (unrounded).
    """
    d = Q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    Kr = rope_rows(K, np.arange(K.shape[0]), rope_dims, base)
    V = f64(V)
    out = {}
    for t in rows:
        p = q_start + t
        q = rope_rows(f64(Q[t])[None], np.array([p]), rope_dims, base)[0]   # [H, d]
        lo = max(0, p - window + 1)
        s = (q @ Kr[lo:p + 1].T) * scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        out[t] = (e / e.sum(axis=1, keepdims=True)) @ V[lo:p + 1]
    return out


# ---------------------------------------------------------------------------
# Decode over the FP8 cache
# ---------------------------------------------------------------------------

def dequant_cache(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """k_j = E4M3(code_j) * scale_j, exact in fp64."""
    return e4m3_decode(u8(codes)) * f64(scales)[:, None]


def decode_select(Q: np.ndarray, Kc: np.ndarray, Vc: np.ndarray, ks: np.ndarray,
                  vs: np.ndarray, seqs: Sequence[int], kv_len: int, window: int,
                  topk: int, scale: Optional[float] = None) -> Dict[int, SelectRow]:
    """Decode: the cache of sequence b holds kv_len tokens, the new token's own
    K/V included; its query sits at position kv_len-1 and sees keys [0, kv_len)."""
    d = Q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = {}
    for b in seqs:
        K = dequant_cache(Kc[b, :kv_len], ks[b, :kv_len])
        V = dequant_cache(Vc[b, :kv_len], vs[b, :kv_len])
        out[b] = select_row(f64(Q[b]), K, V, kv_len - 1,
                            window, topk, scale)
    return out


def sparse_attn_decode(Qs: np.ndarray, Kc: np.ndarray, Vc: np.ndarray, ks: np.ndarray,
                       vs: np.ndarray, idx: np.ndarray, seqs: Sequence[int],
                       scale: Optional[float] = None) -> Dict[int, np.ndarray]:
    """Sparse layer at decode over the FP8 cache: sequence b's query attends to
    the rows idx[b] of its OWN cache, key row j being E4M3(Kc[b,j]) * ks[b,j]
    and value row j being E4M3(Vc[b,j]) * vs[b,j]."""
    d = Qs.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    idx = idx.cpu().numpy() if hasattr(idx, "cpu") else np.asarray(idx)
    out = {}
    for b in seqs:
        row = np.asarray(idx[b])
        S = row[row >= 0].astype(np.int64)
        K = dequant_cache(u8(Kc[b])[S], f64(ks[b])[S])
        V = dequant_cache(u8(Vc[b])[S], f64(vs[b])[S])
        local = np.arange(S.shape[0], dtype=np.int32)
        out[b] = sparse_attn_row(f64(Qs[b]), K, V, local, scale)
    return out
