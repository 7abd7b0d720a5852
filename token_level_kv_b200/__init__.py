"""Python binding of libhs2.so -- the HySparse2 token-level KV Reuse hot path
on B200 (sm_100a).

Argument marshalling only: shapes are read off the tensors, pointers and the
current CUDA stream are passed to the C ABI (include/hs2.h), and a non-zero
status is raised as Hs2Error.  Every step of the computation runs in the
library's CUDA kernels; there is no other code path.  PyTorch is used for
device memory and streams.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs2.so")

KV_BF16 = 0
KV_FP8_E4M3 = 1

STATUS = {0: "HS2_OK", 1: "HS2_ERR_INVALID_ARG", 2: "HS2_ERR_UNSUPPORTED", 3: "HS2_ERR_WORKSPACE",
          4: "HS2_ERR_CUDA", 5: "HS2_ERR_TIMEOUT", 6: "HS2_ERR_DEVICE_CHECK"}


class Hs2Error(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python token_level_kv_b200/build.py` "
                          "(nvcc, sm_100a); there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, L, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "hs2_status_string": ([I], ctypes.c_char_p),
        "hs2_last_error": ([], ctypes.c_char_p),
        "hs2_version": ([], ctypes.c_char_p),
        "hs2_bridge_kv": ([P, L, I, P, P, I, I, P, P, P, P, P], I),
        "hs2_bridge_append": ([P, I, I, P, P, I, P, P, P, P, L, P, P], I),
        "hs2_full_attn_select": ([P, P, P, P, P, I, I, L, L, L, L, I, I, I, I, F, P, P, P, Z, P], I),
        "hs2_full_attn_select_blocks": ([P, P, P, P, P, I, I, L, L, L, L, I, I, I, I, I, F, P, P, P, Z, P], I),
        "hs2_full_attn_select_workspace": ([I, I, L, L, I, I, I, I, ctypes.POINTER(Z)], I),
        "hs2_sparse_attn_prefill": ([P, P, P, P, L, L, I, I, I, F, P, P], I),
        "hs2_sparse_attn_decode": ([P, P, P, P, P, I, I, L, L, P, I, I, I, F, P, P, Z, P], I),
        "hs2_sparse_attn_decode_workspace": ([I, I, I, I, ctypes.POINTER(Z)], I),
        "hs2_sparse_attn_decode_static": ([P, P, P, P, P, I, I, L, L, P, I, I, I, F, P, P], I),
        "hs2_swa_attn_prefill": ([P, P, P, L, L, L, I, I, I, I, F, F, P, P, Z, P], I),
        "hs2_swa_attn_prefill_workspace": ([L, L, I, I, I, ctypes.POINTER(Z)], I),
        "hs2_decode_shard_workspace": ([I, L, I, I, I, I, ctypes.POINTER(Z)], I),
        "hs2_decode_shard_attn": ([P, P, P, P, P, I, L, L, I, I, I, F, P, P, P, Z, P], I),
        "hs2_partial_merge": ([P, I, I, P, P, I, I, I, P], I),
        "hs2_partial_finalize": ([P, P, P, I, I, I, P], I),
        "hs2_decode_shard_candidates": ([P, Z, I, L, L, L, I, I, I, I, P, P, P], I),
        "hs2_decode_merge_candidates": ([P, I, I, L, I, I, P, P], I),
        "hs2_sparse_decode_shard": ([P, P, P, P, P, I, L, L, L, P, I, I, I, F, P, P, P, Z, P], I),
        "hs2_device_status": ([P], I),
        "hs2_set_spin_limit": ([L], I),
        "hs2_profile_enable": ([I], I),
        "hs2_profile_collect": ([ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(F), I, ctypes.POINTER(I)], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


lib = _load()
EXPORTS = ("hs2_status_string", "hs2_last_error", "hs2_version", "hs2_bridge_kv", "hs2_full_attn_select",
           "hs2_full_attn_select_workspace", "hs2_sparse_attn_prefill", "hs2_sparse_attn_decode",
           "hs2_sparse_attn_decode_workspace", "hs2_device_status", "hs2_set_spin_limit",
           "hs2_profile_enable", "hs2_profile_collect", "hs2_sparse_attn_decode_static", "hs2_bridge_append",
           "hs2_full_attn_select_blocks", "hs2_swa_attn_prefill", "hs2_swa_attn_prefill_workspace",
           "hs2_decode_shard_workspace", "hs2_decode_shard_attn", "hs2_partial_merge", "hs2_partial_finalize",
           "hs2_decode_shard_candidates", "hs2_decode_merge_candidates", "hs2_sparse_decode_shard")


def _check(status: int) -> None:
    if status != 0:
        raise Hs2Error(status, lib.hs2_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("hs2 takes device tensors only (got a CPU tensor)")
    if not t.is_contiguous():
        raise ValueError("hs2 takes contiguous tensors only")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _kv_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KV_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return KV_FP8_E4M3
    raise ValueError(f"K/V must be bf16 or FP8 E4M3 codes, got {t.dtype}")


def hs2_version() -> str:
    return lib.hs2_version().decode()


def hs2_bridge_kv(hidden, Wk, Wv, K_out, V_out, k_scale=None, v_scale=None, stream=None) -> None:
    """K_out = hidden Wk^T, V_out = hidden Wv^T; FP8 codes + row scales when K_out is uint8."""
    rows, D = hidden.shape
    d = Wk.shape[0]
    out = _kv_dtype(K_out)
    _check(lib.hs2_bridge_kv(_ptr(hidden), rows, D, _ptr(Wk), _ptr(Wv), d, out, _ptr(K_out), _ptr(V_out),
                             _ptr(k_scale), _ptr(v_scale), _stream(stream)))


def hs2_bridge_append(hidden, Wk, Wv, Kc, Vc, k_scale, v_scale, pos, stream=None) -> None:
    """Bridge each sequence's new token (hidden [B, D]) and write its FP8 K/V row
    and scales at row pos[b] of the caches Kc, Vc [B, stride, d], k_scale, v_scale [B, stride]."""
    B, D = hidden.shape
    d = Wk.shape[0]
    if Kc.dim() != 3 or Kc.shape[0] != B or k_scale.shape != Kc.shape[:2]:
        raise ValueError("caches must be [B, stride, d] with scales [B, stride]")
    _check(lib.hs2_bridge_append(_ptr(hidden), B, D, _ptr(Wk), _ptr(Wv), d, _ptr(Kc), _ptr(Vc), _ptr(k_scale),
                                 _ptr(v_scale), Kc.shape[1], _ptr(pos), _stream(stream)))


def hs2_full_attn_select_workspace(kv_dtype: int, batch: int, Tq: int, kv_len: int, Hq: int, d: int,
                                   window: int, topk: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.hs2_full_attn_select_workspace(kv_dtype, batch, Tq, kv_len, Hq, d, window, topk, ctypes.byref(n)))
    return n.value


def hs2_full_attn_select(Q, K, V, O, idx, workspace, *, window: int, topk: int, q_start: int = 0,
                         kv_len: int | None = None, k_scale=None, v_scale=None,
                         softmax_scale: float | None = None, stream=None) -> None:
    """Full-attention layer + token selection.

    prefill (bf16 K/V): Q [Tq, H, d], K/V [>= kv_len, d], O [Tq, H, d], idx [Tq, window+topk].
    decode (FP8 K/V codes): Q [B, H, d], K/V [B, stride, d], k/v_scale [B, stride],
    O [B, H, d], idx [B, window+topk]; the query sits at kv_len - 1.
    """
    a = _select_args(Q, K, q_start, kv_len, softmax_scale, workspace)
    _check(lib.hs2_full_attn_select(_ptr(Q), _ptr(K), _ptr(V), _ptr(k_scale), _ptr(v_scale), a["kvd"], a["batch"],
                                    a["q_start"], a["Tq"], a["kv_len"], a["stride"], a["H"], a["d"], window, topk,
                                    a["scale"], _ptr(O), _ptr(idx), _ptr(workspace), a["ws"], _stream(stream)))


def hs2_full_attn_select_blocks(Q, K, V, O, idx, workspace, *, window: int, block: int, topk_blocks: int,
                                q_start: int = 0, kv_len: int | None = None, k_scale=None, v_scale=None,
                                softmax_scale: float | None = None, stream=None) -> None:
    """Full-attention layer + block-level selection: as hs2_full_attn_select with
    idx [rows, window + topk_blocks * block] holding the chosen blocks' positions."""
    a = _select_args(Q, K, q_start, kv_len, softmax_scale, workspace)
    _check(lib.hs2_full_attn_select_blocks(_ptr(Q), _ptr(K), _ptr(V), _ptr(k_scale), _ptr(v_scale), a["kvd"],
                                           a["batch"], a["q_start"], a["Tq"], a["kv_len"], a["stride"], a["H"], a["d"],
                                           window, block, topk_blocks, a["scale"], _ptr(O), _ptr(idx),
                                           _ptr(workspace), a["ws"], _stream(stream)))


def _select_args(Q, K, q_start, kv_len, softmax_scale, workspace) -> dict:
    kvd = _kv_dtype(K)
    d = Q.shape[-1]
    H = Q.shape[-2]
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    if kvd == KV_BF16:
        batch, Tq = 1, Q.shape[0]
        kv_len = K.shape[0] if kv_len is None else kv_len
        stride = kv_len
    else:
        batch, Tq = Q.shape[0], 1
        stride = K.shape[1]
        kv_len = stride if kv_len is None else kv_len
        q_start = kv_len - 1
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return dict(kvd=kvd, d=d, H=H, scale=scale, batch=batch, Tq=Tq, kv_len=kv_len, stride=stride, q_start=q_start,
                ws=ws)


def hs2_swa_attn_prefill_workspace(Tq: int, kv_len: int, Hq: int, d: int, rope_dims: int = 64) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.hs2_swa_attn_prefill_workspace(Tq, kv_len, Hq, d, rope_dims, ctypes.byref(n)))
    return n.value


def hs2_swa_attn_prefill(Q, K, V, O, workspace, *, window: int, q_start: int = 0, kv_len: int | None = None,
                         rope_dims: int = 64, rope_base: float = 10000.0, softmax_scale: float | None = None,
                         stream=None) -> None:
    """Sliding-window attention with partial RoPE: Q [Tq, H, d] at positions
    q_start.. over K, V [>= kv_len, d]; O [Tq, H, d]."""
    Tq, H, d = Q.shape
    kv_len = K.shape[0] if kv_len is None else kv_len
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.hs2_swa_attn_prefill(_ptr(Q), _ptr(K), _ptr(V), q_start, Tq, kv_len, H, d, window, rope_dims,
                                    rope_base, scale, _ptr(O), _ptr(workspace), ws, _stream(stream)))


def hs2_sparse_attn_prefill(Q, K, V, idx, O, *, kv_len: int | None = None, softmax_scale: float | None = None,
                            stream=None) -> None:
    """Sparse layer: Q [Tq, H, d] over the rows idx [Tq, n_idx] of the shared K/V [kv_len, d]."""
    Tq, H, d = Q.shape
    kv_len = K.shape[0] if kv_len is None else kv_len
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    _check(lib.hs2_sparse_attn_prefill(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), Tq, kv_len, idx.shape[-1], H, d,
                                       scale, _ptr(O), _stream(stream)))


def hs2_sparse_attn_decode_workspace(batch: int, n_idx: int, Hq: int, d: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.hs2_sparse_attn_decode_workspace(batch, n_idx, Hq, d, ctypes.byref(n)))
    return n.value


def hs2_sparse_attn_decode(Q, Kc, Vc, k_scale, v_scale, idx, O, workspace=None, *, kv_len: int | None = None,
                           softmax_scale: float | None = None, stream=None) -> None:
    """Sparse layer over the FP8 cache: Q [B, H, d], Kc/Vc [B, stride, d] codes, idx [B, n_idx]."""
    B, H, d = Q.shape
    stride = Kc.shape[1]
    kv_len = stride if kv_len is None else kv_len
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.hs2_sparse_attn_decode(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(k_scale), _ptr(v_scale), KV_FP8_E4M3, B,
                                      kv_len, stride, _ptr(idx), idx.shape[-1], H, d, scale, _ptr(O),
                                      _ptr(workspace), ws, _stream(stream)))


def hs2_sparse_attn_decode_static(Q, Kc, Vc, k_scale, v_scale, idx, O, *, kv_len: int | None = None,
                                  softmax_scale: float | None = None, stream=None) -> None:
    """hs2_sparse_attn_decode for callers that cannot allocate device memory:
    the split partials go to the library's own 8 MiB static device array
    instead of a workspace.  Calls that overlap on the GPU share that array
    and race; run them one after another."""
    B, H, d = Q.shape
    stride = Kc.shape[1]
    kv_len = stride if kv_len is None else kv_len
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    _check(lib.hs2_sparse_attn_decode_static(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(k_scale), _ptr(v_scale),
                                             KV_FP8_E4M3, B, kv_len, stride, _ptr(idx), idx.shape[-1], H, d,
                                             scale, _ptr(O), _stream(stream)))


# ---- decode with the context split over shards (one per GPU); the exchanges
# between the calls are the caller's (token_level_kv_b200.sharded runs them
# over torch.distributed)

def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def hs2_decode_shard_workspace(batch: int, shard_len: int, n_idx: int, Hq: int, d: int, topk: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.hs2_decode_shard_workspace(batch, shard_len, n_idx, Hq, d, topk, ctypes.byref(n)))
    return n.value


def candidates_numel(batch: int, topk: int) -> int:
    """4-byte elements of one shard's candidate block: scores, positions, lengths."""
    return 2 * batch * topk + batch


def hs2_decode_shard_attn(Q, Kc, Vc, k_scale, v_scale, ml_out, O_out, workspace, *, topk: int,
                          shard_len: int | None = None, softmax_scale: float | None = None, stream=None) -> None:
    """Full attention over one shard: ml_out fp32 [2, B, H] (m, l), O_out fp32 [B, H, d] unnormalised."""
    B, H, d = Q.shape
    stride = Kc.shape[1]
    n = stride if shard_len is None else shard_len
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    _check(lib.hs2_decode_shard_attn(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(k_scale), _ptr(v_scale), B, n, stride, H,
                                     d, topk, scale, _ptr(ml_out), _ptr(O_out), _ptr(workspace),
                                     _nbytes(workspace), _stream(stream)))


def hs2_partial_merge(ml_all, shard: int, O32, ml_out, stream=None) -> None:
    """ml_all fp32 [R, 2, B, H]; rescales O32 [B, H, d] in place; ml_out fp32 [B, H, 2] = (M, L)."""
    R, _, B, H = ml_all.shape
    _check(lib.hs2_partial_merge(_ptr(ml_all), R, shard, _ptr(O32), _ptr(ml_out), B, H, O32.shape[-1],
                                 _stream(stream)))


def hs2_partial_finalize(ml, O32, O, stream=None) -> None:
    """O bf16 [B, H, d] = O32 / L."""
    B, H, d = O32.shape
    _check(lib.hs2_partial_finalize(_ptr(ml), _ptr(O32), _ptr(O), B, H, d, _stream(stream)))


def hs2_decode_shard_candidates(workspace, ml_global, cand, *, batch: int, shard_len: int, shard_offset: int,
                                kv_len: int, Hq: int, d: int, window: int, topk: int, stream=None) -> None:
    """The shard's top-k candidates under the global (M, L) into cand (candidates_numel 4-byte elements)."""
    _check(lib.hs2_decode_shard_candidates(_ptr(workspace), _nbytes(workspace), batch, shard_len, shard_offset,
                                           kv_len, Hq, d, window, topk, _ptr(ml_global), _ptr(cand),
                                           _stream(stream)))


def hs2_decode_merge_candidates(cand_all, idx, *, kv_len: int, window: int, topk: int, stream=None) -> None:
    """cand_all [R, candidates_numel]; idx int32 [B, window + topk]."""
    R = cand_all.shape[0]
    B = idx.shape[0]
    _check(lib.hs2_decode_merge_candidates(_ptr(cand_all), R, B, kv_len, window, topk, _ptr(idx), _stream(stream)))


def hs2_sparse_decode_shard(Q, Kc, Vc, k_scale, v_scale, idx, ml_out, O_out, workspace, *, shard_offset: int,
                            shard_len: int | None = None, softmax_scale: float | None = None,
                            stream=None) -> None:
    """A sparse layer over one shard: the entries of idx (global positions) the shard holds."""
    B, H, d = Q.shape
    stride = Kc.shape[1]
    n = stride if shard_len is None else shard_len
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    _check(lib.hs2_sparse_decode_shard(_ptr(Q), _ptr(Kc), _ptr(Vc), _ptr(k_scale), _ptr(v_scale), B, n, stride,
                                       shard_offset, _ptr(idx), idx.shape[-1], H, d, scale, _ptr(ml_out),
                                       _ptr(O_out), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def hs2_device_status(stream=None) -> int:
    """Synchronises the stream; returns the device status (0 = OK) and clears it."""
    return lib.hs2_device_status(_stream(stream))


def hs2_set_spin_limit(iterations: int) -> None:
    _check(lib.hs2_set_spin_limit(iterations))


def hs2_profile_enable(on: bool) -> None:
    """Bracket every library kernel launch of this host thread with CUDA events."""
    _check(lib.hs2_profile_enable(1 if on else 0))


def hs2_profile_collect(max_n: int = 4096):
    """[(kernel name, device ms)] for the launches recorded since enable; clears the record."""
    names = (ctypes.c_char_p * max_n)()
    ms = (ctypes.c_float * max_n)()
    n = ctypes.c_int(0)
    _check(lib.hs2_profile_collect(names, ms, max_n, ctypes.byref(n)))
    return [(names[i].decode(), float(ms[i])) for i in range(min(n.value, max_n))]


def workspace(nbytes: int, device="cuda") -> torch.Tensor | None:
    """A 256-byte aligned device buffer of at least nbytes (None for 0)."""
    if nbytes == 0:
        return None
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
