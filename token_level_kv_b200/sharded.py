"""Decode with each sequence's context split over the ranks of a process group.

For the 1M-token regime with few sequences (agihunt.info summary, KV cache
table at 1M tokens) one GPU's decode is a handful of CTAs per sequence and
the cache may not fit one GPU; here rank q holds positions
[offset_q, offset_q + len_q) of every sequence's FP8 cache, the ranks' ranges
tiling [0, kv_len) in rank order.  One decode step of a full-attention layer
(the exact selector) and its sparse layers is the library's per-shard calls
with three kinds of exchange between them:

  full attention   hs2_decode_shard_attn          -> (m, l) and unnormalised O
                   all-gather (m, l)              -> every shard's (m, l)
                   hs2_partial_merge              -> global (M, L); O rescaled
                   all-reduce (sum) O             -> hs2_partial_finalize: O
  selection        hs2_decode_shard_candidates    -> the shard's top-k list
                   all-gather the lists           -> hs2_decode_merge_candidates
  sparse layers    hs2_sparse_decode_shard        -> (m, l, O) over the index
                   entries the shard holds, then the same merge as above.

The exchanges are tiny (B*H*2 floats, B*k candidates, B*H*d floats), so the
step's time is the shards' kernels plus a few collective latencies.  The
index row and the outputs equal those of the single-GPU calls on the whole
cache, up to the order of fp32 additions in the merged sums (the index row
exactly, but for selection scores within rounding of the k-th one).

Argument marshalling only: every step of the arithmetic runs in the
library's kernels, the exchanges in the process group's collectives (NCCL
over NVLink on GPUs).
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import (candidates_numel, hs2_decode_merge_candidates, hs2_decode_shard_attn, hs2_decode_shard_candidates,
               hs2_decode_shard_workspace, hs2_partial_finalize, hs2_partial_merge, hs2_sparse_decode_shard,
               workspace)


def shard_bounds(kv_len: int, n_shards: int, align: int = 64) -> list[tuple[int, int]]:
    """(offset, length) of each shard: whole units of `align` positions
    (1 when the context is shorter than one unit per shard) spread evenly,
    the last shard also taking the ragged tail."""
    if n_shards < 1 or kv_len < n_shards:
        raise ValueError(f"cannot split {kv_len} positions over {n_shards} shards")
    if kv_len < n_shards * align:
        align = 1
    units = kv_len // align
    sizes = [(units // n_shards + (1 if q < units % n_shards else 0)) * align for q in range(n_shards)]
    sizes[-1] += kv_len - units * align
    offs = [sum(sizes[:q]) for q in range(n_shards)]
    return list(zip(offs, sizes))


class LibraryOps:
    """The per-shard steps: the library's calls (the default)."""
    shard_attn = staticmethod(hs2_decode_shard_attn)
    partial_merge = staticmethod(hs2_partial_merge)
    partial_finalize = staticmethod(hs2_partial_finalize)
    shard_candidates = staticmethod(hs2_decode_shard_candidates)
    merge_candidates = staticmethod(hs2_decode_merge_candidates)
    sparse_shard = staticmethod(hs2_sparse_decode_shard)

    @staticmethod
    def workspace_bytes(batch, shard_len, n_idx, Hq, d, topk):
        return hs2_decode_shard_workspace(batch, shard_len, n_idx, Hq, d, topk)

    @staticmethod
    def workspace(nbytes, device):
        return workspace(nbytes, device)


class GroupExchange:
    """The exchanges over a torch.distributed process group, one local shard
    per rank: all-gather into one flat buffer, all-reduce with SUM."""

    def __init__(self, group=None):
        self.group = group
        self.n_shards = dist.get_world_size(group)

    def all_gather(self, local: list[torch.Tensor]) -> torch.Tensor:
        (t,) = local
        out = torch.empty(self.n_shards * t.numel(), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.reshape(-1), group=self.group)
        return out.view(self.n_shards, *t.shape)

    def all_reduce_sum(self, local: list[torch.Tensor]) -> None:
        (t,) = local
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)


class _Shard:
    def __init__(self, q, offset, length, B, H, d, k, n_idx, ops, device):
        self.q, self.offset, self.length = q, offset, length
        self.ml = torch.empty(2, B, H, dtype=torch.float32, device=device)
        self.O32 = torch.empty(B, H, d, dtype=torch.float32, device=device)
        self.cand = torch.empty(candidates_numel(B, k), dtype=torch.int32, device=device)
        self.ws = ops.workspace(ops.workspace_bytes(B, length, n_idx, H, d, k), device)


class ShardedDecode:
    """One decode step over context shards.  `shards` names the shards this
    process holds: its rank alone under a process group (GroupExchange), or
    every shard when one process runs them all with an exchange of its own.

      step(Q, caches, Q_sparse) -> (O, idx, [O_sparse])
        Q bf16 [B, H, d] (the full layer's query), Q_sparse: the sparse
        layers' queries; caches[i] = (Kc, Vc, k_scale, v_scale) of local
        shard i: codes uint8 [B, stride, d], scales fp32 [B, stride], local
        row r = global position offset + r.  O bf16 [B, H, d] and idx int32
        [B, window + topk] (global positions) are the same on every shard.
        idx is this object's buffer: the next step overwrites it (the O
        tensors are new each step).
    """

    def __init__(self, *, kv_len: int, n_shards: int, shards: list[int], batch: int, Hq: int, d: int,
                 window: int = 128, topk: int = 1024, exchange, ops=LibraryOps, device="cuda",
                 bounds: list[tuple[int, int]] | None = None, softmax_scale: float | None = None):
        self.bounds = bounds if bounds is not None else shard_bounds(kv_len, n_shards)
        if len(self.bounds) != n_shards or self.bounds[0][0] != 0 or sum(n for _, n in self.bounds) != kv_len or \
                any(self.bounds[i][0] + self.bounds[i][1] != self.bounds[i + 1][0] for i in range(n_shards - 1)):
            raise ValueError("the shards must tile [0, kv_len) in order")
        self.kv_len, self.n_shards = kv_len, n_shards
        self.B, self.H, self.d, self.window, self.topk = batch, Hq, d, window, topk
        self.scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
        self.ex, self.ops, self.device = exchange, ops, device
        self.local = [_Shard(q, *self.bounds[q], batch, Hq, d, topk, window + topk, ops, device) for q in shards]
        self.mlg = torch.empty(batch, Hq, 2, dtype=torch.float32, device=device)
        self.idx = torch.empty(batch, window + topk, dtype=torch.int32, device=device)

    def _merge(self) -> torch.Tensor:
        """(m, l, O) of every shard -> the normalised output, on every shard."""
        ml_all = self.ex.all_gather([s.ml for s in self.local])
        for s in self.local:
            self.ops.partial_merge(ml_all, s.q, s.O32, self.mlg)
        self.ex.all_reduce_sum([s.O32 for s in self.local])
        O = torch.empty(self.B, self.H, self.d, dtype=torch.bfloat16, device=self.device)
        self.ops.partial_finalize(self.mlg, self.local[0].O32, O)
        return O

    def step(self, Q, caches, Q_sparse=()):
        if len(caches) != len(self.local):
            raise ValueError(f"{len(caches)} caches for {len(self.local)} local shards")
        for s, c in zip(self.local, caches):
            self.ops.shard_attn(Q, *c, s.ml, s.O32, s.ws, topk=self.topk, shard_len=s.length,
                                softmax_scale=self.scale)
        O = self._merge()
        # self.mlg now holds the full layer's global (M, L): the selection scores' normaliser
        for s in self.local:
            self.ops.shard_candidates(s.ws, self.mlg, s.cand, batch=self.B, shard_len=s.length,
                                      shard_offset=s.offset, kv_len=self.kv_len, Hq=self.H, d=self.d,
                                      window=self.window, topk=self.topk)
        cand_all = self.ex.all_gather([s.cand for s in self.local])
        self.ops.merge_candidates(cand_all, self.idx, kv_len=self.kv_len, window=self.window, topk=self.topk)
        outs = []
        for Qs in Q_sparse:
            for s, c in zip(self.local, caches):
                self.ops.sparse_shard(Qs, *c, self.idx, s.ml, s.O32, s.ws, shard_offset=s.offset,
                                      shard_len=s.length, softmax_scale=self.scale)
            outs.append(self._merge())
        return O, self.idx, outs
