"""Parity rules between the CUDA path and the fp64 oracle (test code).

Index sets (one row): the forced-window segment must be bit-exact; the
selection segment must be ascending, -1 padded, inside the candidate range,
free of duplicates and the same size as the oracle's; every key in the
symmetric difference must score within ``rel`` of the oracle's k-th largest
score tau (oracle scores).  Several sets are correct when scores tie; this is
the part that is unique.

Outputs: max-abs error against the unrounded oracle, 2e-2 with bf16 KV and
6e-2 with FP8 KV (fp32 accumulation on the GPU).
"""
from __future__ import annotations

import numpy as np

TOL_BF16 = 2e-2
TOL_FP8 = 6e-2
TIE_REL = 1e-6


def check_idx_row(gpu_row, ora, window: int, topk: int, rel: float = TIE_REL):
    """Returns (ok, n_swaps, message) for one row; ``ora`` is an oracle SelectRow."""
    g = np.asarray(gpu_row).astype(np.int64)
    o = ora.idx.astype(np.int64)
    if g.shape != o.shape:
        return False, 0, f"shape {g.shape} vs {o.shape}"
    if not np.array_equal(g[:window], o[:window]):
        return False, 0, f"window segment differs at p={ora.p}"
    gs = g[window:]
    n = int((gs >= 0).sum())
    if n != ora.n_sel:
        return False, 0, f"p={ora.p}: {n} selected vs oracle {ora.n_sel}"
    if not np.all(gs[n:] == -1) or not np.all(gs[:n] >= 0):
        return False, 0, f"p={ora.p}: selection not packed then -1 padded"
    sel = gs[:n]
    if n > 1 and not np.all(np.diff(sel) > 0):
        return False, 0, f"p={ora.p}: selection not strictly ascending"
    n_cand = max(0, ora.p - window + 1)
    if n and (sel[-1] >= n_cand):
        return False, 0, f"p={ora.p}: selected key {sel[-1]} inside the window"
    so = set(o[window:window + ora.n_sel].tolist())
    sg = set(sel.tolist())
    diff = so ^ sg
    if not diff:
        return True, 0, ""
    if ora.tau is None:
        return False, len(diff), f"p={ora.p}: all candidates must be taken"
    tau = ora.tau
    for j in diff:
        if abs(ora.sigma[j] - tau) > rel * tau:
            return False, len(diff), (f"p={ora.p}: key {j} sigma={ora.sigma[j]:.10g} "
                                      f"tau={tau:.10g} outside the tie margin")
    return True, len(diff) // 2, ""


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def check_block_row(gpu_row, ora_blk, window: int, block: int, topk_blocks: int, rel: float = TIE_REL):
    """Block-level rows: window bit-exact; the selection is whole candidate
    blocks (each block's candidate positions, consecutive), ascending, then -1;
    the chosen block set equals the oracle's except for blocks whose score lies
    within ``rel`` of the oracle's k-th largest block score.  ``ora_blk`` is an
    oracle BlockSelectRow.  Returns (ok, n_swaps, message)."""
    g = np.asarray(gpu_row).astype(np.int64)
    o = ora_blk.idx.astype(np.int64)
    p = ora_blk.p
    if g.shape != o.shape:
        return False, 0, f"shape {g.shape} vs {o.shape}"
    if not np.array_equal(g[:window], o[:window]):
        return False, 0, f"window segment differs at p={p}"
    sel = g[window:]
    n = int((sel >= 0).sum())
    if not np.all(sel[:n] >= 0) or not np.all(sel[n:] == -1):
        return False, 0, f"p={p}: selection not packed then -1 padded"
    n_cand = max(0, p - window + 1)
    blocks = []
    i = 0
    while i < n:
        c = int(sel[i] // block)
        want = np.arange(c * block, min(n_cand, (c + 1) * block))
        if want.size == 0 or not np.array_equal(sel[i:i + want.size], want):
            return False, 0, f"p={p}: block {c} not emitted whole at slot {i}"
        if blocks and c <= blocks[-1]:
            return False, 0, f"p={p}: blocks not ascending"
        blocks.append(c)
        i += want.size
    nb = ora_blk.block_score.shape[0]
    if len(blocks) != min(topk_blocks, nb):
        return False, 0, f"p={p}: {len(blocks)} blocks vs {min(topk_blocks, nb)}"
    diff = set(blocks) ^ set(ora_blk.blocks.tolist())
    if not diff:
        return True, 0, ""
    if ora_blk.tau is None:
        return False, len(diff), f"p={p}: all blocks must be taken"
    for c in diff:
        if abs(ora_blk.block_score[c] - ora_blk.tau) > rel * ora_blk.tau:
            return False, len(diff), (f"p={p}: block {c} score={ora_blk.block_score[c]:.10g} "
                                      f"tau={ora_blk.tau:.10g} outside the tie margin")
    return True, len(diff) // 2, ""
