"""Seeded synthetic inputs for the HySparse2 KV Reuse hot path.

This module is the only code shared by the CUDA path (tests, bench) and the
fp64 oracle.  It draws numbers and lays them out in the shapes the method's
workloads have; it holds none of the method's arithmetic (no attention, no
selection, no bridging, no quantiser of its own -- FP8 cache bytes for the
decode workloads come from torch's built-in ``float8_e4m3fn`` cast).

Generator (counter based, so any element can be drawn on its own):

* ``bits(seed, stream, i)`` = splitmix64-mix(key(seed, stream) + (i+1)*phi),
  with phi = 0x9E3779B97F4A7C15 and key = mix(seed*0xD1B54A32D192ED03 + stream),
  all in wrapping 64-bit arithmetic.  splitmix64's finaliser is Steele,
  Lea & Flood, "Fast splittable pseudorandom number generators" (OOPSLA 2014).
* uniform u in [0,1): (bits >> 11) * 2^-53 (53-bit dyadic).
* standard normal for element e: Box-Muller on counters 2e and 2e+1 in fp64,
  z = sqrt(-2 ln(1-u0)) cos(2 pi u1).
* bf16 values are the fp64 draw times a scale, rounded by torch's cast.

The same tensor is always generated once and handed to both sides (the
oracle gets a CPU copy), so the two never depend on libm agreeing across
devices.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

_PHI = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_SEED_MUL = 0xD1B54A32D192ED03
_MASK64 = (1 << 64) - 1

# one stream id per tensor kind
STREAMS = {
    "q_full": 1, "k": 2, "v": 3, "needle": 4, "zipf": 5, "hidden": 6,
    "kv_scale_k": 7, "kv_scale_v": 8, "q_sparse": 100, "wk": 200, "wv": 300,
    "q_bridged": 400,
}


def _s64(x: int) -> int:
    """Python int -> the int64 with the same low 64 bits."""
    x &= _MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


def _mix_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 lanes viewed as uint64."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _s64(_M1)
    z = (z ^ _srl(z, 27)) * _s64(_M2)
    return z ^ _srl(z, 31)


def stream_key(seed: int, stream: int) -> int:
    return _mix_int(seed * _SEED_MUL + stream)


def bits(seed: int, stream: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """``count`` 64-bit draws (as int64) for counters start..start+count-1."""
    key = stream_key(seed, stream)
    ctr = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    return _mix(ctr * _s64(_PHI) + _s64(key))


def uniform(seed: int, stream: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """fp64 uniforms in [0, 1) on a 2^-53 grid."""
    return _srl(bits(seed, stream, start, count, device), 11).to(torch.float64) * (2.0 ** -53)


def normal(seed: int, stream: int, count: int, device="cpu", start: int = 0,
           chunk: int = 1 << 26) -> torch.Tensor:
    """fp64 standard normals, element e from counters 2(start+e), 2(start+e)+1."""
    out = torch.empty(count, dtype=torch.float64, device=device)
    for c0 in range(0, count, chunk):
        n = min(chunk, count - c0)
        u = uniform(seed, stream, 2 * (start + c0), 2 * n, device).view(n, 2)
        r = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))
        out[c0:c0 + n] = r * torch.cos((2.0 * math.pi) * u[:, 1])
        del u, r
    return out


def normal_bf16(seed: int, stream: int, shape, scale: float = 1.0, device="cpu") -> torch.Tensor:
    n = 1
    for s in shape:
        n *= s
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    chunk = 1 << 26
    for c0 in range(0, n, chunk):
        m = min(chunk, n - c0)
        out[c0:c0 + m] = (normal(seed, stream, m, device, start=c0) * scale).to(torch.bfloat16)
    return out.view(*shape)


def randint(seed: int, stream: int, start: int, count: int, lo: int, hi: int) -> List[int]:
    """Integers uniform in [lo, hi] (inclusive) by floor(u*(hi-lo+1))."""
    u = uniform(seed, stream, start, count)
    return [lo + min(int(math.floor(x * (hi - lo + 1))), hi - lo) for x in u.tolist()]


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

@dataclass
class PrefillCase:
    """Inputs of one full-attention+select layer and its sparse layers."""
    T: int
    H: int
    d: int
    window: int
    topk: int
    Q: torch.Tensor            # bf16 [T, H, d]  full layer's queries
    K: torch.Tensor            # bf16 [T, d]     the one KV head
    V: torch.Tensor            # bf16 [T, d]
    Q_sparse: List[torch.Tensor]   # bf16 [T, H, d] per sparse layer
    needles: List[Tuple[int, int]] = field(default_factory=list)  # (key pos, target row)
    chunk: Optional[int] = None

    @property
    def n_idx(self) -> int:
        return self.window + self.topk


def plant_needles(Q: torch.Tensor, K: torch.Tensor, n: int, seed: int, window: int,
                  logit: float = 8.0) -> List[Tuple[int, int]]:
    """Overwrite n key rows so that each lines up with one later query row.

    Needle m: key position p uniform in [0, T-1-window], target row i uniform in
    [p+window, T-1]; K[p] = c * qbar/|qbar| with qbar the mean over heads of
    Q[i], c chosen so that mean_h(q_ih . K[p])/sqrt(d) = ``logit``.
    """
    T, H, d = Q.shape
    out = []
    for m in range(n):
        (p,) = randint(seed, STREAMS["needle"], 4 * m, 1, 0, T - 1 - window)
        (i,) = randint(seed, STREAMS["needle"], 4 * m + 1, 1, p + window, T - 1)
        qbar = Q[i].to(torch.float64).mean(dim=0)
        nrm = torch.linalg.vector_norm(qbar)
        k = qbar * (logit * math.sqrt(d) / (nrm * nrm))
        K[p] = k.to(device=K.device, dtype=K.dtype)
        out.append((p, i))
    return out


def zipf_key_norms(T: int, seed: int, device="cpu", top: float = 6.0) -> torch.Tensor:
    """n_j = max(1, top * r_j^-1/2) for a seeded random rank permutation r."""
    keys = bits(seed, STREAMS["zipf"], 0, T, device)
    order = torch.argsort(keys)
    rank = torch.empty(T, dtype=torch.float64, device=device)
    rank[order] = torch.arange(1, T + 1, dtype=torch.float64, device=device)
    return torch.clamp(top / torch.sqrt(rank), min=1.0)


def make_prefill_case(T: int, H: int, d: int, window: int, topk: int, n_sparse: int,
                      n_needles: int = 0, scale: float = 1.0, zipf: bool = False,
                      seed: int = 0, device="cpu", chunk: Optional[int] = None) -> PrefillCase:
    Q = normal_bf16(seed, STREAMS["q_full"], (T, H, d), scale, device)
    if zipf:
        nrm = zipf_key_norms(T, seed, device)
        K = torch.empty(T, d, dtype=torch.bfloat16, device=device)
        for r0 in range(0, T, 1 << 16):
            r1 = min(T, r0 + (1 << 16))
            z = normal(seed, STREAMS["k"], (r1 - r0) * d, device, start=r0 * d).view(r1 - r0, d)
            K[r0:r1] = (z * (scale * nrm[r0:r1, None])).to(torch.bfloat16)
    else:
        K = normal_bf16(seed, STREAMS["k"], (T, d), scale, device)
    V = normal_bf16(seed, STREAMS["v"], (T, d), scale, device)
    needles = plant_needles(Q, K, n_needles, seed, window) if n_needles else []
    Qs = [normal_bf16(seed, STREAMS["q_sparse"] + l, (T, H, d), scale, device)
          for l in range(n_sparse)]
    return PrefillCase(T, H, d, window, topk, Q, K, V, Qs, needles, chunk)


@dataclass
class DecodeCase:
    """One new query per sequence over an FP8 E4M3 cache with per-token scales."""
    B: int
    N: int
    H: int
    d: int
    window: int
    topk: int
    Q: torch.Tensor            # bf16 [B, H, d]
    Kc: torch.Tensor           # uint8 (E4M3 codes) [B, N, d]
    Vc: torch.Tensor           # uint8 [B, N, d]
    ks: torch.Tensor           # fp32 [B, N]
    vs: torch.Tensor           # fp32 [B, N]
    Q_sparse: List[torch.Tensor]

    @property
    def n_idx(self) -> int:
        return self.window + self.topk


def fp8_rows_from_normal(seed: int, stream: int, B: int, N: int, d: int, device="cpu",
                         rows_per_chunk: int = 1 << 18):
    """E4M3 codes + per-row fp32 scales of bf16 N(0,1) rows.

    scale = amax/448 of the bf16 row (1 if the row is all zero) in fp32; codes are
    torch's own float8_e4m3fn cast of row/scale.
    """
    R = B * N
    codes = torch.empty(R, d, dtype=torch.uint8, device=device)
    scales = torch.empty(R, dtype=torch.float32, device=device)
    for r0 in range(0, R, rows_per_chunk):
        r1 = min(R, r0 + rows_per_chunk)
        x = normal(seed, stream, (r1 - r0) * d, device, start=r0 * d).to(torch.bfloat16)
        x = x.view(r1 - r0, d).to(torch.float32)
        amax = x.abs().amax(dim=1)
        sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        codes[r0:r1] = (x / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        scales[r0:r1] = sc
    return codes.view(B, N, d), scales.view(B, N)


def make_decode_case(B: int, N: int, H: int, d: int, window: int, topk: int, n_sparse: int,
                     seed: int = 0, device="cpu") -> DecodeCase:
    Q = normal_bf16(seed, STREAMS["q_full"], (B, H, d), 1.0, device)
    Kc, ks = fp8_rows_from_normal(seed, STREAMS["k"], B, N, d, device)
    Vc, vs = fp8_rows_from_normal(seed, STREAMS["v"], B, N, d, device)
    Qs = [normal_bf16(seed, STREAMS["q_sparse"] + l, (B, H, d), 1.0, device)
          for l in range(n_sparse)]
    return DecodeCase(B, N, H, d, window, topk, Q, Kc, Vc, ks, vs, Qs)


@dataclass
class BridgeCase:
    """Self-decoder hidden states and per-layer bridging projections ([out, in])."""
    hidden: torch.Tensor       # bf16 [R, D]
    Wk: List[torch.Tensor]     # bf16 [d, D] per cross-decoder full layer
    Wv: List[torch.Tensor]


def make_bridge_case(R: int, D: int, d: int, n_layers: int, seed: int = 0,
                     device="cpu") -> BridgeCase:
    hidden = normal_bf16(seed, STREAMS["hidden"], (R, D), 1.0, device)
    ws = 1.0 / math.sqrt(D)
    Wk = [normal_bf16(seed, STREAMS["wk"] + l, (d, D), ws, device) for l in range(n_layers)]
    Wv = [normal_bf16(seed, STREAMS["wv"] + l, (d, D), ws, device) for l in range(n_layers)]
    return BridgeCase(hidden, Wk, Wv)


def bridged_decode_queries(B: int, H: int, d: int, n_layers: int, n_sparse: int, seed: int = 0,
                           device="cpu") -> List[Tuple[torch.Tensor, List[torch.Tensor]]]:
    """Per cross-decoder layer l: its full layer's new-token queries and those of
    its n_sparse sparse layers, bf16 N(0,1) [B, H, d] (stream q_bridged + 10*l + i)."""
    out = []
    for l in range(n_layers):
        base = STREAMS["q_bridged"] + 10 * l
        q = normal_bf16(seed, base, (B, H, d), 1.0, device)
        out.append((q, [normal_bf16(seed, base + 1 + i, (B, H, d), 1.0, device) for i in range(n_sparse)]))
    return out


# The five workloads (sizes from the method's own regimes: 32k pretraining,
# 256k post-training, 1M evaluation).
CONFIGS = {
    1: dict(kind="prefill", T=1024, H=8, d=128, window=128, topk=256, n_sparse=1,
            n_needles=4, scale=1.0),
    2: dict(kind="prefill", T=32768, H=16, d=256, window=128, topk=1024, n_sparse=3,
            n_needles=64, scale=1.0 / 16.0),
    3: dict(kind="decode", B=64, N=131072, H=16, d=256, window=128, topk=1024, n_sparse=3),
    4: dict(kind="prefill", T=262144, H=16, d=256, window=128, topk=1024, n_sparse=2,
            n_needles=0, scale=1.0, zipf=True, chunk=8192),
    5: dict(kind="bridged_decode", B=4, N=1 << 20, H=16, d=256, D=2048, window=128,
            topk=1024, n_layers=2, n_sparse=3),
}
