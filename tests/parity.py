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
