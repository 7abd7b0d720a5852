"""CPU stand-ins (test code) for the library's per-shard decode calls, written
from their contracts in include/hs2.h in float64 with the oracle's FP8
decoding, so that the orchestration in token_level_kv_b200.sharded -- shard
bounds, the order and shapes of the exchanges, the global offsets -- can run
over gloo ranks without a GPU.  Buffers are the same torch tensors the
library's calls take, on the CPU; the workspace is a dict that keeps the
shard's logits between the attention and the candidate calls."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

LOG2E = 1.0 / math.log(2.0)


def _f64(t):
    return t.detach().to(torch.float64).numpy()


def _attend(q, K, V, scale):
    """(m, l, O) of one query's heads over rows K, V in log2 units; -inf, 0, 0 without rows."""
    H, d = q.shape
    if K.shape[0] == 0:
        return np.full(H, -np.inf), np.zeros(H), np.zeros((H, d)), np.zeros((H, 0))
    x = (q @ K.T) * scale * LOG2E
    m = x.max(axis=1)
    p = np.exp2(x - m[:, None])
    return m, p.sum(axis=1), p @ V, x


class CpuOps:
    @staticmethod
    def workspace_bytes(batch, shard_len, n_idx, Hq, d, topk):
        return 1

    @staticmethod
    def workspace(nbytes, device):
        return {}

    @staticmethod
    def shard_attn(Q, Kc, Vc, k_scale, v_scale, ml_out, O_out, ws, *, topk, shard_len=None, softmax_scale=None):
        B, H, d = Q.shape
        n = Kc.shape[1] if shard_len is None else shard_len
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
        for b in range(B):
            K = oracle.dequant_cache(Kc[b, :n].numpy(), k_scale[b, :n].numpy())
            V = oracle.dequant_cache(Vc[b, :n].numpy(), v_scale[b, :n].numpy())
            m, l, O, x = _attend(_f64(Q[b]), K, V, scale)
            ml_out[0, b] = torch.from_numpy(m)
            ml_out[1, b] = torch.from_numpy(l)
            O_out[b] = torch.from_numpy(O)
            ws[b] = x

    @staticmethod
    def partial_merge(ml_all, shard, O32, ml_out):
        m, l = _f64(ml_all[:, 0]), _f64(ml_all[:, 1])          # [R, B, H]
        M = m.max(axis=0)
        w = np.where(np.isneginf(m), 0.0, np.exp2(m - M[None]))
        O32 *= torch.from_numpy(w[shard]).to(O32.dtype)[..., None]
        ml_out[..., 0] = torch.from_numpy(M)
        ml_out[..., 1] = torch.from_numpy((l * w).sum(axis=0))

    @staticmethod
    def partial_finalize(ml, O32, O):
        L = _f64(ml[..., 1])[..., None]
        O.copy_(torch.from_numpy(np.where(L > 0, _f64(O32) / np.where(L > 0, L, 1.0), 0.0)))

    @staticmethod
    def shard_candidates(ws, ml_global, cand, *, batch, shard_len, shard_offset, kv_len, Hq, d, window, topk):
        k = topk
        val = cand[:batch * k].view(torch.float32).view(batch, k)
        pos = cand[batch * k:2 * batch * k].view(batch, k)
        cnt = cand[2 * batch * k:]
        n = max(0, min(shard_len, kv_len - window - shard_offset))
        M, L = _f64(ml_global[..., 0]), _f64(ml_global[..., 1])
        for b in range(batch):
            sig = (np.exp2(ws[b][:, :n] - M[b][:, None]) / L[b][:, None]).sum(axis=0) if n else np.zeros(0)
            sel = oracle.topk_positions(sig, k)
            val[b, :sel.shape[0]] = torch.from_numpy(sig[sel])
            pos[b, :sel.shape[0]] = torch.from_numpy(sel + shard_offset)
            cnt[b] = sel.shape[0]

    @staticmethod
    def merge_candidates(cand_all, idx, *, kv_len, window, topk):
        R = cand_all.shape[0]
        B = idx.shape[0]
        k = topk
        for b in range(B):
            vals, poss = [], []
            for r in range(R):
                c = int(cand_all[r, 2 * B * k + b])
                vals.append(cand_all[r, b * k:b * k + c].view(torch.float32).double().numpy())
                poss.append(cand_all[r, B * k + b * k:B * k + b * k + c].numpy().astype(np.int64))
            v, p = np.concatenate(vals), np.concatenate(poss)
            take = np.sort(p[np.lexsort((p, -v))[:k]])
            row = np.full(window + k, -1, dtype=np.int32)
            row[:window] = oracle.window_slots(kv_len - 1, window)
            row[window:window + take.shape[0]] = take
            idx[b] = torch.from_numpy(row)

    @staticmethod
    def sparse_shard(Q, Kc, Vc, k_scale, v_scale, idx, ml_out, O_out, ws, *, shard_offset, shard_len=None,
                     softmax_scale=None):
        B, H, d = Q.shape
        n = Kc.shape[1] if shard_len is None else shard_len
        scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
        for b in range(B):
            row = idx[b].numpy().astype(np.int64)
            S = row[(row >= shard_offset) & (row < shard_offset + n)] - shard_offset
            K = oracle.dequant_cache(Kc[b].numpy()[S], k_scale[b].numpy()[S])
            V = oracle.dequant_cache(Vc[b].numpy()[S], v_scale[b].numpy()[S])
            m, l, O, _ = _attend(_f64(Q[b]), K, V, scale)
            ml_out[0, b] = torch.from_numpy(m)
            ml_out[1, b] = torch.from_numpy(l)
            O_out[b] = torch.from_numpy(O)
