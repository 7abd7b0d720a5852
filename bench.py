#!/usr/bin/env python
"""Benchmark of the HySparse2 token-level KV Reuse hot path on B200.

One step = one pass of the prefill hot path over the paper-shape workload:
T = 32768 queries, 16 heads, one KV head, d = 256, bf16 N(0,1)/16 inputs with
64 planted needles; the full-attention layer with selection (window 128 +
top-1024 -> int32 [T, 1152]) followed by 3 sparse layers reusing the index set
and the KV.  The value is the step's algorithmic TFLOP/s (full attention
4*d*H*T(T+1)/2 plus the sparse layers 4*d*H*sum_t |S_t|) over all ranks.

The same line also carries the decode step over an FP8 cache (64 sequences of
131072 tokens: full attention + selection, then 3 sparse layers, L2 flushed
before each sparse call) and the KV Bridging GEMM of the 1M-token bridged
decode workload (4 x 2^20 hidden rows, 2 layers), each with its roofline.

--impl reference times the fp64 CPU oracle on sampled rows of the same
workload (the reference arm: there is no other implementation to run).

Launch: python bench.py --gpus N --steps K --warmup W  (N > 1 under torchrun;
every rank runs its own copy of the workload: weak scaling, no collective on
the data path).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "sparse-attn decode tok/s & HBM GB/s; full-attn+top-k prefill TFLOP/s vs peak"
WORKLOAD = dict(T=32768, H=16, d=256, window=128, topk=1024, n_sparse=3, n_needles=64, scale=1.0 / 16.0)
DECODE = dict(B=64, N=131072, H=16, d=256, window=128, topk=1024, n_sparse=3)
BRIDGE = dict(R=4 * (1 << 20), D=2048, d=256, layers=2)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def visible_gpu_index(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        return vis.split(",")[local_rank].strip()
    return str(local_rank)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons every 200 ms while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-i", gpu, "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = []
        for ln in open(self.f.name):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5], parts[6], parts[7],
                             parts[8]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        pmax = max(r[2] for r in rows)
        load = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in load:
            for n, v in zip(names, r[3:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": pmax}


# ---------------------------------------------------------------------------
# workload arithmetic
# ---------------------------------------------------------------------------

def dram_traffic(kernel: str):
    """DRAM bytes per query row of one launch of `kernel`, from the ncu capture
    recorded in profiles/dram_traffic.json, or None when there is none or when
    the kernel's source has changed since (its SHA-256 no longer matches)."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))[kernel]
        src = open(os.path.join(ROOT, rec["source"]), "rb").read()
    except (OSError, KeyError, ValueError):
        return None, None
    if hashlib.sha256(src).hexdigest() != rec["sha256"]:
        return None, f"stale: {rec['source']} changed since the capture"
    return rec["dram_bytes"] / rec["rows"], rec["note"]


def prefill_flops(T, H, d, window, topk, n_sparse):
    full = 4.0 * d * H * T * (T + 1) / 2                       # QK^T and PV over the causal pairs
    n_idx = window + topk
    sel = sum(min(p + 1, n_idx) for p in range(T))              # |S_t| (window + selected)
    sparse = 4.0 * d * H * sel
    sigma = 2.0 * d * H * sum(max(0, p - window + 1) for p in range(T))   # QK^T again, candidates only
    return full, sparse, n_sparse * sparse, sigma


def reduce_max(value: float, device) -> float:
    """Max over all ranks (the timing rule for N > 1); works for nccl and gloo."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(step_flops: float, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs one replica of the step."""
    return world * step_flops / (max_ms * 1e-3) / 1e12


def timed_steps(step, steps, flush, stream):
    """Per-step CUDA events on the launching stream, L2 flushed between steps."""
    ts = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ts]


def warm_up(step, n=3, seconds=0.3):
    """At least n untimed steps and at least `seconds` of them: a measurement
    that follows a power-capped GEMM phase starts once the SM clock has come
    back (right after the bridging GEMM the clock sat near half its maximum
    for tens of milliseconds, doubling the decode kernels' times)."""
    t0 = time.perf_counter()
    i = 0
    while i < n or time.perf_counter() - t0 < seconds:
        step()
        i += 1
        if i % 4 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()


def graph_step_ms(step, n, flush, stream):
    """The step captured once as a CUDA graph and replayed (L2 flushed before
    each replay): the launch gaps between its kernels go away."""
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()                                   # warm on the capture stream
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    ms = statistics.median(timed_steps(g.replay, n, flush, stream))
    del g
    return ms


def per_kernel(records):
    agg = {}
    for name, ms in records:
        c = agg.setdefault(name, [0, 0.0])
        c[0] += 1
        c[1] += ms
    return {k: {"launches": v[0], "total_ms": v[1], "avg_ms": v[1] / v[0]} for k, v in agg.items()}


# ---------------------------------------------------------------------------
# oracle on sampled rows (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

class OracleSample:
    def __init__(self, case, seed=0):
        import numpy as np
        import oracle
        self.np, self.oracle = np, oracle
        self.case = case
        self.Kc = oracle.f64(case.K.cpu())
        self.Vc = oracle.f64(case.V.cpu())
        self.Q = case.Q.cpu()
        self.Qs = [q.cpu() for q in case.Q_sparse]
        self.rng = np.random.default_rng(seed)

    def run_rows(self, n_rows):
        c = self.case
        rows = sorted(int(x) for x in self.rng.integers(0, c.T, size=n_rows))
        t0 = time.perf_counter()
        ref = self.oracle.full_attn_select(self.Q, self.Kc, self.Vc, rows, 0, c.window, c.topk)
        flops = 0.0
        for t in rows:
            idx = ref[t].idx
            for q in self.Qs:
                self.oracle.sparse_attn_row(self.oracle.f64(q[t]), self.Kc, self.Vc, idx, 1.0 / math.sqrt(c.d))
            flops += 4.0 * c.d * c.H * (t + 1) + len(self.Qs) * 4.0 * c.d * c.H * int((idx >= 0).sum())
        return flops, time.perf_counter() - t0, len(rows)


def host_cores() -> int:
    """Cores this process may run on (its affinity mask)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def oracle_threads() -> int:
    """Let the oracle's BLAS use every core of the affinity mask and return the
    thread count it then runs with (the cores the CPU baseline actually used)."""
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        threadpool_limits(limits=host_cores(), user_api="blas")
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args):
    import synth
    w = WORKLOAD
    case = synth.make_prefill_case(w["T"], w["H"], w["d"], w["window"], w["topk"], w["n_sparse"],
                                   n_needles=w["n_needles"], scale=w["scale"], seed=0, device="cpu")
    cores = oracle_threads()
    smp = OracleSample(case, seed=1)
    rows_per_step = args.ref_rows
    for _ in range(args.warmup):
        smp.run_rows(max(1, rows_per_step // 4))
    fl, tt, nr = 0.0, 0.0, 0
    for _ in range(args.steps):
        f, t, n = smp.run_rows(rows_per_step)
        fl, tt, nr = fl + f, tt + t, nr + n
    value = fl / tt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(), "sample": f"{rows_per_step} seeded rows per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "affinity_cores": host_cores(),
                         "kind": "oracle",
                         "sample": f"{nr} sampled query rows of the workload (full attention + selection + "
                                   f"3 sparse layers each), {tt:.1f} s", "cpu": cpu_model()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_name():
    w = WORKLOAD
    return (f"prefill T={w['T']} H={w['H']} d={w['d']} MQA NoPE, window {w['window']} + top-{w['topk']}, "
            f"{w['n_sparse']} sparse layers, bf16 N(0,1)/16 + {w['n_needles']} needles")


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, dist):
    import synth
    import token_level_kv_b200 as hs2

    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()
    if args.sharded_nccl:
        flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        res = bench_sharded_nccl(hs2, dev, stream, lambda: flush_buf.zero_(), args, rank, world)
        if rank == 0:
            print(json.dumps({"decode_1m_sharded_nccl": res}), flush=True)
        return
    if args.only_decode:
        flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)

        def flush_only():
            flush_buf.zero_()
            flush_rd.max()
        if rank == 0:
            print(json.dumps({"decode": bench_decode(hs2, dev, stream, flush_only, peaks, peak_src, args)}), flush=True)
        return
    w = WORKLOAD
    T, H, d, W, k = w["T"], w["H"], w["d"], w["window"], w["topk"]
    case = synth.make_prefill_case(T, H, d, W, k, w["n_sparse"], n_needles=w["n_needles"], scale=w["scale"],
                                   seed=0, device=dev)
    O = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(T, W + k, dtype=torch.int32, device=dev)
    Os = [torch.empty_like(O) for _ in range(w["n_sparse"])]
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_BF16, 1, T, T, H, d, W, k), dev)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush():
        # write 256 MiB (> 126 MB L2), then read another 256 MiB so the timed
        # call does not pay for writing the flush's dirty lines back
        flush_buf.zero_()
        flush_rd.max()

    def step():
        hs2.hs2_full_attn_select(case.Q, case.K, case.V, O, idx, ws, window=W, topk=k)
        for l in range(w["n_sparse"]):
            hs2.hs2_sparse_attn_prefill(case.Q_sparse[l], case.K, case.V, idx, Os[l])

    full_fl, sparse_fl1, sparse_fl, sigma_fl = prefill_flops(T, H, d, W, k, w["n_sparse"])
    step_flops = full_fl + sparse_fl

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = hs2.hs2_device_status()
    if st != 0:
        raise RuntimeError(f"device status {hs2.STATUS.get(st)} after warm-up")

    sampler = ClockSampler(visible_gpu_index(int(os.environ.get("LOCAL_RANK", 0)))) if rank == 0 else None
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    hs2.hs2_profile_enable(True)
    t_wall = time.perf_counter()
    step_ms = timed_steps(step, args.steps, flush, stream)
    t_wall = time.perf_counter() - t_wall
    prof = hs2.hs2_profile_collect()
    hs2.hs2_profile_enable(False)
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    ms = statistics.mean(step_ms)
    if dist:
        ms = reduce_max(ms, dev)
    value = weak_scaling_value(step_flops, world, ms)
    kern = per_kernel(prof)
    launches = len(prof)

    # roofline of the dominant kernel and of the whole full-attention + selection call
    dom = max(kern, key=lambda n: kern[n]["total_ms"])
    # algorithmic tensor work per launch; the sparse layer's unique HBM bytes
    # (Q, O, idx, K, V: ~0.7 GB) take less time at the HBM roofline than its
    # FLOPs at the tensor roofline, so its bound is the tensor one
    work = {"fa_fwd_kernel": full_fl, "select_sigma_kernel": sigma_fl, "sparse_prefill_kernel": sparse_fl1,
            "sparse_tc_kernel": sparse_fl1}
    roof = None
    if dom in work:
        ach = work[dom] / (kern[dom]["avg_ms"] * 1e-3) / 1e12
        tr, tr_note = dram_traffic(dom)
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                "traffic": tr * T if tr is not None else None,
                "traffic_source": tr_note,
                "peak_source": f"{peak_src} bf16_tflops (burst: kernels of a few ms, timed one by one)"}
    sel_ms = sum(kern.get(n, {"avg_ms": 0.0})["avg_ms"] for n in ("fa_fwd_kernel", "select_sigma_kernel",
                                                                  "topk_select_kernel"))
    sel_ach = full_fl / (sel_ms * 1e-3) / 1e12 if sel_ms > 0 else None
    # ---------------- the same call with block-level selection (64-token blocks, 16 of them)
    blocks = bench_select_blocks(hs2, case, ws, flush, stream, full_fl, peaks) if not args.no_blocks else None
    stages = {n: {"avg_ms": v["avg_ms"], "launches": v["launches"], "share": v["total_ms"] / sum(
        x["total_ms"] for x in kern.values())} for n, v in kern.items()}

    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_name(), "global_batch": world, "seq_len": T,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "flushed between steps (256 MiB write); K/V (33.5 MB) stay L2-resident within a step",
                   "flops_per_step": step_flops},
        "roofline": roof,
        "select_call": {"ms": sel_ms, "achieved_tflops": sel_ach, "frac": (sel_ach or 0) / peaks["bf16_tflops"],
                        "algorithmic_flops": full_fl, "executed_extra_flops_sigma_pass": sigma_fl,
                        "unit": "TFLOP/s", "peak": peaks["bf16_tflops"]},
        "stages": stages,
        "select_blocks": blocks,
        "gpu_launches": launches,
        "wall_s_timed_region": t_wall,
    }

    # ---------------- end to end through the public API with host buffers
    if not args.no_e2e:
        hin = [t.cpu().pin_memory() for t in [case.Q, case.K, case.V] + case.Q_sparse]
        din = [torch.empty_like(t, device=dev) for t in hin]
        hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in [O, idx] + Os]
        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in hout)
        # the step in query chunks over the causal prefix (the calls' chunked
        # form; the same work and bit-identical results), so that results
        # start leaving while later chunks compute
        C = next((c for c in (16, 8, 4) if T % c == 0 and T // c >= 2048), 1)   # 16 at T = 32768: 27.9 ms, 8: 28.4, 4: 29.5, 1: 38.3
        Tc = T // C
        ws_c = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_BF16, 1, Tc, T, H, d, W, k), dev)

        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

        def e2e_step():
            # every step copies all of its inputs in and all of its results out;
            # the copies run on their own streams (PCIe is full duplex), in the
            # order the chunks need them, and each chunk's results leave as soon
            # as they are complete
            main = torch.cuda.current_stream()
            s_in.wait_stream(main)                 # the previous step no longer reads din
            ev_in = []
            with torch.cuda.stream(s_in):
                for h, dd in zip(hin[1:3], din[1:3]):          # K, V
                    dd.copy_(h, non_blocking=True)
                for c in range(C):
                    r = slice(c * Tc, (c + 1) * Tc)
                    evs = []
                    for j in [0] + [3 + l for l in range(w["n_sparse"])]:
                        din[j][r].copy_(hin[j][r], non_blocking=True)
                        evs.append(torch.cuda.Event())
                        evs[-1].record(s_in)
                    ev_in.append(evs)
            for c in range(C):
                r = slice(c * Tc, (c + 1) * Tc)
                main.wait_event(ev_in[c][0])
                hs2.hs2_full_attn_select(din[0][r], din[1], din[2], O[r], idx[r], ws_c, window=W, topk=k,
                                         q_start=c * Tc, kv_len=(c + 1) * Tc)
                s_out.wait_stream(main)
                with torch.cuda.stream(s_out):
                    hout[0][r].copy_(O[r], non_blocking=True)
                    hout[1][r].copy_(idx[r], non_blocking=True)
                for l in range(w["n_sparse"]):
                    main.wait_event(ev_in[c][1 + l])
                    hs2.hs2_sparse_attn_prefill(din[3 + l][r], din[1], din[2], idx[r], Os[l][r])
                    s_out.wait_stream(main)
                    with torch.cuda.stream(s_out):
                        hout[2 + l][r].copy_(Os[l][r], non_blocking=True)
            main.wait_stream(s_out)                # the step ends with every result on the host
            main.wait_stream(s_in)

        e2e_step()
        torch.cuda.synchronize()
        e_ms = statistics.mean(timed_steps(e2e_step, max(2, min(args.steps, 5)), lambda: None, stream))
        if dist:
            e_ms = reduce_max(e_ms, dev)
        out["e2e"] = {"value": weak_scaling_value(step_flops, world, e_ms), "unit": "TFLOP/s", "ms_per_step": e_ms,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "copies": "pinned host buffers; inputs in and results out on their own streams, "
                                "overlapped with the step's kernels",
                      "chunks": f"{C} query chunks of {Tc} over the causal prefix"}
        del hin, din, hout

    # ---------------- decode over the FP8 cache
    if not args.no_decode:
        out["decode"] = bench_decode(hs2, dev, stream, flush, peaks, peak_src, args)
    # ---------------- KV Bridging GEMM, then the bridged 1M-token decode step over its caches
    if not args.no_bridge:
        out["bridge"], bridged = bench_bridge(hs2, dev, stream, flush, peaks, peak_src)
        if not args.no_decode:
            out["decode_1m"] = bench_bridged_decode(hs2, dev, stream, flush, peaks, peak_src, args, bridged)
            out["decode_1m_sharded"] = bench_sharded_decode(hs2, dev, stream, flush, args, bridged)
        del bridged
        torch.cuda.empty_cache()
    # ---------------- the 1M decode with the context split over the ranks (NCCL exchanges)
    if dist and not args.no_decode:
        out["decode_1m_sharded_nccl"] = bench_sharded_nccl(hs2, dev, stream, flush, args, rank, world)
        torch.cuda.empty_cache()
    # ---------------- chunked prefill at 256k and the tiny launch-bound case
    if not args.no_long:
        out["prefill_256k"] = bench_prefill_256k(hs2, dev, stream, peaks, peak_src, args)
        torch.cuda.empty_cache()
    out["prefill_1k"] = bench_tiny(hs2, dev, stream, flush, args)
    out["swa_32k"] = bench_swa(hs2, case, flush, stream, peaks)
    out["select_call_frac"] = {"prefill_32k": out["select_call"]["frac"],
                               "prefill_256k_chunked": out.get("prefill_256k", {}).get("select_call_frac"),
                               "peak": f"{peak_src} bf16_tflops", "target": 0.60}

    clocks = sampler.stop() if sampler else None
    st = hs2.hs2_device_status()
    if st != 0:
        raise RuntimeError(f"device status {hs2.STATUS.get(st)} after the timed region")

    # ---------------- oracle on the host cores (rank 0, one GPU only)
    if rank == 0:
        out["clocks"] = clocks
        if world == 1 and not args.no_cpu:
            cores = oracle_threads()
            smp = OracleSample(case, seed=2)
            fl, tt, nr = 0.0, 0.0, 0
            while tt < args.cpu_seconds:
                f, t, n = smp.run_rows(16)
                fl, tt, nr = fl + f, tt + t, nr + n
            out["cpu_baseline"] = {"value": fl / tt / 1e12, "unit": "TFLOP/s", "cores": cores,
                                   "affinity_cores": host_cores(),
                                   "kind": "oracle", "cpu": cpu_model(),
                                   "sample": f"{nr} seeded query rows of the workload (full attention + "
                                             f"selection + 3 sparse layers per row), {tt:.1f} s"}
        print(json.dumps(out), flush=True)


def bench_decode(hs2, dev, stream, flush, peaks, peak_src, args):
    import synth
    c = DECODE
    B, N, H, d, W, k = c["B"], c["N"], c["H"], c["d"], c["window"], c["topk"]
    dc = synth.make_decode_case(B, N, H, d, W, k, c["n_sparse"], seed=0, device=dev)
    O = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(B, W + k, dtype=torch.int32, device=dev)
    Os = torch.empty_like(O)
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_FP8_E4M3, B, 1, N, H, d, W, k), dev)
    wss = hs2.workspace(hs2.hs2_sparse_attn_decode_workspace(B, W + k, H, d), dev)

    def full():
        hs2.hs2_full_attn_select(dc.Q, dc.Kc, dc.Vc, O, idx, ws, window=W, topk=k, k_scale=dc.ks, v_scale=dc.vs)

    def sparse(l):
        hs2.hs2_sparse_attn_decode(dc.Q_sparse[l], dc.Kc, dc.Vc, dc.ks, dc.vs, idx, Os, wss)

    def warm_step():
        full()
        for l in range(c["n_sparse"]):
            sparse(l)

    warm_up(warm_step)
    n = max(3, args.steps)
    hs2.hs2_profile_enable(True)
    t_full = timed_steps(full, n, flush, stream)
    prof_full = per_kernel(hs2.hs2_profile_collect())
    t_sp = [timed_steps(lambda l=l: sparse(l), n, flush, stream) for l in range(c["n_sparse"])]
    prof_sp = per_kernel(hs2.hs2_profile_collect())
    hs2.hs2_profile_enable(False)
    t_warm = timed_steps(lambda: [sparse(l) for l in range(c["n_sparse"])], n, lambda: None, stream)

    def whole_step():
        full()
        for l in range(c["n_sparse"]):
            sparse(l)
    g_ms = graph_step_ms(whole_step, n, flush, stream)
    prof = {"full_select_call": prof_full, "sparse_call": prof_sp}
    ms_full = statistics.median(t_full)
    ms_sp = [statistics.median(t) for t in t_sp]
    # device time of the sparse-decode kernels alone (library events around each launch)
    sp_kernel_ms = sum(v["total_ms"] for v in prof_sp.values()) / (n * c["n_sparse"])
    full_bytes = B * N * (2 * d + 8) + B * H * d * 2 * 2 + B * (W + k) * 4
    sp_bytes = B * ((W + k) * (2 * d + 8 + 4) + 2 * H * d * 2)
    step_ms = ms_full + sum(ms_sp)
    sp_gbs = sp_bytes / (statistics.mean(ms_sp) * 1e-3) / 1e9
    full_gbs = full_bytes / (ms_full * 1e-3) / 1e9
    return {
        "workload": f"decode B={B} N={N} H={H} d={d} FP8 E4M3 cache + per-token scales, "
                    f"window {W} + top-{k}, 3 sparse layers",
        "tok_s": B / (step_ms * 1e-3), "step_ms": step_ms,
        "step_ms_cuda_graph": g_ms, "tok_s_cuda_graph": B / (g_ms * 1e-3),
        "full_select_ms": ms_full, "full_select_gbs": full_gbs, "full_select_frac": full_gbs / peaks["hbm_gbs"],
        "sparse_ms": ms_sp, "sparse_gbs": sp_gbs, "sparse_frac": sp_gbs / peaks["hbm_gbs"],
        "sparse_kernel_ms": sp_kernel_ms,
        "sparse_kernel_gbs": sp_bytes / (sp_kernel_ms * 1e-3) / 1e9,
        "sparse_kernel_frac": sp_bytes / (sp_kernel_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "sparse_tok_s_per_layer": B / (statistics.mean(ms_sp) * 1e-3),
        "sparse_warm_chain_ms": statistics.median(t_warm),
        "algorithmic_bytes": {"full_select": full_bytes, "sparse_per_layer": sp_bytes},
        "l2": "flushed before every timed call (warm chain: the 3 sparse layers back to back, not flushed)",
        "peak": peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm_gbs", "kernels": prof,
    }


def bench_select_blocks(hs2, case, ws, flush, stream, full_fl, peaks, block=64, topk_blocks=16):
    """The full-attention layer with block-level selection on the same inputs:
    aligned 64-token blocks scored by their summed selection scores, the top
    16 taken (the pages' token-vs-block ablation at the same 1024 budget)."""
    T, H, d = case.Q.shape
    W = WORKLOAD["window"]
    O = torch.empty(T, H, d, dtype=torch.bfloat16, device=case.Q.device)
    idx = torch.empty(T, W + block * topk_blocks, dtype=torch.int32, device=case.Q.device)

    def call():
        hs2.hs2_full_attn_select_blocks(case.Q, case.K, case.V, O, idx, ws, window=W, block=block,
                                        topk_blocks=topk_blocks)

    for _ in range(2):
        call()
    torch.cuda.synchronize()
    hs2.hs2_profile_enable(True)
    t = timed_steps(call, 3, flush, stream)
    prof = per_kernel(hs2.hs2_profile_collect())
    hs2.hs2_profile_enable(False)
    ms = statistics.median(t)
    return {"workload": f"as the step's full layer, block-level selection: {topk_blocks} blocks of {block} tokens",
            "ms": ms, "frac": full_fl / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "kernels": {k: v["avg_ms"] for k, v in prof.items()}}


def bench_bridge(hs2, dev, stream, flush, peaks, peak_src):
    """KV Bridging of 4 x 2^20 hidden rows into 2 layers' FP8 caches; returns
    the result and the caches (the bridged decode step reads them)."""
    import synth
    c = BRIDGE
    R, D, d, L = c["R"], c["D"], c["d"], c["layers"]
    bc = synth.make_bridge_case(R, D, d, L, seed=0, device=dev)
    bc_w = list(zip(bc.Wk, bc.Wv))
    Ks = [torch.empty(R, d, dtype=torch.uint8, device=dev) for _ in range(L)]
    Vs = [torch.empty(R, d, dtype=torch.uint8, device=dev) for _ in range(L)]
    ks = [torch.empty(R, dtype=torch.float32, device=dev) for _ in range(L)]
    vs = [torch.empty(R, dtype=torch.float32, device=dev) for _ in range(L)]

    def step():
        for l in range(L):
            hs2.hs2_bridge_kv(bc.hidden, bc.Wk[l], bc.Wv[l], Ks[l], Vs[l], ks[l], vs[l])

    step()
    torch.cuda.synchronize()
    hs2.hs2_profile_enable(True)
    t = timed_steps(step, 3, flush, stream)
    prof = per_kernel(hs2.hs2_profile_collect())
    hs2.hs2_profile_enable(False)
    ms = statistics.median(t)
    flops = 2.0 * R * D * (2 * d) * L
    ach = flops / (ms * 1e-3) / 1e12
    res = {"workload": f"KV Bridging {L} layers: hidden bf16 [{R}, {D}] x W_k, W_v [{d}, {D}] -> FP8 K/V + scales",
           "ms": ms, "achieved_tflops": ach, "peak": peaks["bf16_tflops"], "frac": ach / peaks["bf16_tflops"],
           "peak_source": f"{peak_src} bf16_tflops", "kernels": prof}
    # the new token of each sequence (its last position), for the decode step's append
    hid_new = bc.hidden.view(4, R // 4, D)[:, -1].contiguous()
    del bc
    return res, (list(zip(Ks, Vs, ks, vs)), hid_new, bc_w)


def bench_bridged_decode(hs2, dev, stream, flush, peaks, peak_src, args, bridged):
    """The decode step of the 1M-token bridged workload: 4 sequences of 2^20
    tokens, for each of the 2 cross-decoder layers (over the FP8 caches the
    bridging GEMM just wrote) the new token's bridging + FP8 append at position
    N - 1, full attention + selection and 3 sparse layers; L2 flushed before
    each step."""
    import synth
    caches, hid_new, weights = bridged
    c = synth.CONFIGS[5]
    B, H, d, W, k, ns = c["B"], c["H"], c["d"], c["window"], c["topk"], c["n_sparse"]
    N = BRIDGE["R"] // B                          # tokens per sequence of the bridged caches
    qs = synth.bridged_decode_queries(B, H, d, len(caches), ns, seed=0, device=dev)
    O = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
    Os = torch.empty_like(O)
    idx = torch.empty(B, W + k, dtype=torch.int32, device=dev)
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_FP8_E4M3, B, 1, N, H, d, W, k), dev)
    wss = hs2.workspace(hs2.hs2_sparse_attn_decode_workspace(B, W + k, H, d), dev)
    kv = [(K.view(B, N, d), V.view(B, N, d), a.view(B, N), b.view(B, N)) for K, V, a, b in caches]
    pos = torch.full((B,), N - 1, dtype=torch.int32, device=dev)

    def step():
        for (Kc, Vc, ksc, vsc), (Q, Qsp), (Wk, Wv) in zip(kv, qs, weights):
            hs2.hs2_bridge_append(hid_new, Wk, Wv, Kc, Vc, ksc, vsc, pos)
            hs2.hs2_full_attn_select(Q, Kc, Vc, O, idx, ws, window=W, topk=k, k_scale=ksc, v_scale=vsc)
            for Qs in Qsp:
                hs2.hs2_sparse_attn_decode(Qs, Kc, Vc, ksc, vsc, idx, Os, wss)

    warm_up(step)
    n = max(3, args.steps)
    hs2.hs2_profile_enable(True)
    t = timed_steps(step, n, flush, stream)
    prof = per_kernel(hs2.hs2_profile_collect())
    hs2.hs2_profile_enable(False)
    ms = statistics.median(t)
    g_ms = graph_step_ms(step, n, flush, stream)
    L = len(kv)
    full_bytes = B * N * (2 * d + 8)
    sp_bytes = B * ((W + k) * (2 * d + 8 + 4) + 2 * H * d * 2)
    byte_total = L * (full_bytes + ns * sp_bytes)
    return {"workload": f"bridged decode B={B} N={N} H={H} d={d}, {L} layers x (new-token bridging + FP8 append, "
                        f"full + select, {ns} sparse) over the FP8 caches written by the bridging GEMM",
            "step_ms": ms, "tok_s": B / (ms * 1e-3), "gbs": byte_total / (ms * 1e-3) / 1e9,
            "step_ms_cuda_graph": g_ms, "tok_s_cuda_graph": B / (g_ms * 1e-3),
            "frac": byte_total / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "algorithmic_bytes": byte_total,
            "l2": "flushed before each step", "peak": peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm_gbs",
            "kernels": prof}


class _OneProcessExchange:
    """All shards in this process: the all-gather stacks, the all-reduce sums."""

    def all_gather(self, local):
        return torch.stack(local)

    def all_reduce_sum(self, local):
        total = torch.stack(local).sum(0)
        for t in local:
            t.copy_(total)


def bench_sharded_decode(hs2, dev, stream, flush, args, bridged, R=4):
    """The 1M-token decode of one cross-decoder layer (full + select, 3 sparse
    layers) with each sequence's context split over R shards, against the
    same layer on one GPU over the whole cache.  One GPU here: the shards run
    one after another in this process, and what is timed for the sharded
    case is shard 0's own calls (what each GPU of an R-GPU job runs between
    its collectives); the exchanges are listed by size, not timed."""
    import synth
    from token_level_kv_b200 import sharded
    caches, _, _ = bridged
    c = synth.CONFIGS[5]
    B, H, d, W, k, ns = c["B"], c["H"], c["d"], c["window"], c["topk"], c["n_sparse"]
    N = BRIDGE["R"] // B
    Q, Qsp = synth.bridged_decode_queries(B, H, d, 1, ns, seed=0, device=dev)[0]
    K, V, ks, vs = caches[0]
    Kc, Vc, ksc, vsc = K.view(B, N, d), V.view(B, N, d), ks.view(B, N), vs.view(B, N)
    # one GPU, the whole cache
    O = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
    Os = torch.empty_like(O)
    idx = torch.empty(B, W + k, dtype=torch.int32, device=dev)
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_FP8_E4M3, B, 1, N, H, d, W, k), dev)
    wss = hs2.workspace(hs2.hs2_sparse_attn_decode_workspace(B, W + k, H, d), dev)

    def whole():
        hs2.hs2_full_attn_select(Q, Kc, Vc, O, idx, ws, window=W, topk=k, k_scale=ksc, v_scale=vsc)
        for Qs in Qsp:
            hs2.hs2_sparse_attn_decode(Qs, Kc, Vc, ksc, vsc, idx, Os, wss)

    # R shards in this process: one full step fills every exchanged buffer
    sd = sharded.ShardedDecode(kv_len=N, n_shards=R, shards=list(range(R)), batch=B, Hq=H, d=d, window=W, topk=k,
                               exchange=_OneProcessExchange(), device=dev)
    parts = [tuple(t[:, o:o + n].contiguous() for t in (Kc, Vc, ksc, vsc)) for o, n in sd.bounds]
    O_sh, idx_sh, _ = sd.step(Q, parts, Qsp)
    s0, p0 = sd.local[0], parts[0]
    ml_all = torch.stack([s.ml for s in sd.local])
    cand_all = torch.stack([s.cand for s in sd.local])
    mlg = torch.empty(B, H, 2, dtype=torch.float32, device=dev)
    O0 = torch.empty(B, H, d, dtype=torch.bfloat16, device=dev)
    idx0 = torch.empty_like(idx)

    def shard0():
        hs2.hs2_decode_shard_attn(Q, *p0, s0.ml, s0.O32, s0.ws, topk=k, shard_len=s0.length)
        hs2.hs2_partial_merge(ml_all, 0, s0.O32, mlg)
        hs2.hs2_partial_finalize(mlg, s0.O32, O0)
        hs2.hs2_decode_shard_candidates(s0.ws, mlg, s0.cand, batch=B, shard_len=s0.length, shard_offset=0,
                                        kv_len=N, Hq=H, d=d, window=W, topk=k)
        hs2.hs2_decode_merge_candidates(cand_all, idx0, kv_len=N, window=W, topk=k)
        for Qs in Qsp:
            hs2.hs2_sparse_decode_shard(Qs, *p0, idx_sh, s0.ml, s0.O32, s0.ws, shard_offset=0,
                                        shard_len=s0.length)
            hs2.hs2_partial_merge(ml_all, 0, s0.O32, mlg)
            hs2.hs2_partial_finalize(mlg, s0.O32, O0)

    res = {}
    for name, fn in (("one_gpu", whole), ("shard", shard0)):
        warm_up(fn)
        hs2.hs2_profile_enable(True)
        t = timed_steps(fn, max(3, args.steps), flush, stream)
        prof = per_kernel(hs2.hs2_profile_collect())
        hs2.hs2_profile_enable(False)
        res[name] = {"step_ms": statistics.median(t), "step_ms_cuda_graph": graph_step_ms(fn, max(3, args.steps),
                                                                                          flush, stream),
                     "kernels": prof}
    whole()
    agree = float((idx == idx_sh).float().mean())        # differ only where selection scores tie to rounding
    if hs2.hs2_device_status() != 0:
        raise RuntimeError("device status after the sharded decode")
    n_coll = 3 * (1 + ns) + 1
    ex_bytes = (1 + ns) * (R * 2 * B * H * 4 + B * H * d * 4) + R * hs2.candidates_numel(B, k) * 4
    one, sh = res["one_gpu"], res["shard"]
    del parts, sd
    return {"workload": f"decode B={B} N={N} H={H} d={d}: one layer (full + select, {ns} sparse) over the FP8 "
                        f"cache, the context split over {R} shards; shard 0 timed alone on this GPU",
            "shards": R, "one_gpu_step_ms": one["step_ms"], "one_gpu_step_ms_cuda_graph": one["step_ms_cuda_graph"],
            "per_shard_step_ms": sh["step_ms"], "per_shard_step_ms_cuda_graph": sh["step_ms_cuda_graph"],
            "kernel_time_ratio": one["step_ms_cuda_graph"] / sh["step_ms_cuda_graph"],
            "exchange": {"collectives_per_step": n_coll, "bytes_per_rank_per_step": ex_bytes,
                         "kinds": "all-gather (m, l) and sum all-reduce O per layer, all-gather of the "
                                  "candidate lists; not timed (one GPU)"},
            "index_rows_agree_with_one_gpu": agree,
            "kernels_one_gpu": one["kernels"], "kernels_shard": sh["kernels"],
            "l2": "flushed before each step"}


def bench_sharded_nccl(hs2, dev, stream, flush, args, rank, world, warm=20):
    """One layer of the 1M-token decode (4 sequences of 2^20 tokens: full +
    select, 3 sparse layers) with each sequence's context split over the
    world's ranks, one shard per GPU, the exchanges over NCCL (all-gathers of
    (m, l) and of the candidate lists, sum all-reduces of O): device time per
    step, max over ranks.  Every rank runs the same fixed number of steps, so
    the collectives pair up."""
    import synth
    from token_level_kv_b200 import sharded
    c = synth.CONFIGS[5]
    B, N, H, d, W, k, ns = c["B"], c["N"], c["H"], c["d"], c["window"], c["topk"], c["n_sparse"]
    case = synth.make_decode_case(B, N, H, d, W, k, n_sparse=ns, seed=0, device=dev)
    sd = sharded.ShardedDecode(kv_len=N, n_shards=world, shards=[rank], batch=B, Hq=H, d=d, window=W, topk=k,
                               exchange=sharded.GroupExchange(), device=dev)
    off, n = sd.bounds[rank]
    cache = tuple(t[:, off:off + n].contiguous() for t in (case.Kc, case.Vc, case.ks, case.vs))
    Q, Qs = case.Q, list(case.Q_sparse)
    del case
    torch.cuda.empty_cache()

    def step():
        sd.step(Q, [cache], Qs)

    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    torch.distributed.barrier()
    t = timed_steps(step, max(3, args.steps), flush, stream)
    torch.distributed.barrier()
    ms = reduce_max(statistics.median(t), dev)
    if hs2.hs2_device_status() != 0:
        raise RuntimeError("device status after the sharded decode")
    return {"workload": f"decode B={B} N={N} H={H} d={d}: one layer (full + select, {ns} sparse) with the context "
                        f"split over {world} ranks, exchanges over NCCL",
            "shards": world, "shard_len": n, "step_ms": ms, "tok_s": B / (ms * 1e-3),
            "l2": "flushed before each step", "timing": "CUDA events per step, median, max over ranks"}


def bench_prefill_256k(hs2, dev, stream, peaks, peak_src, args):
    """The long chunked prefill: T = 262144, Zipf key norms, the full layer in
    32 query chunks of 8192 over the causal prefix, then 2 sparse layers over
    all rows.  Inputs (2.15 GB of Q alone) are far larger than L2."""
    import synth
    c = synth.CONFIGS[4]
    T, H, d, W, k, ch, ns = c["T"], c["H"], c["d"], c["window"], c["topk"], c["chunk"], c["n_sparse"]
    if args.long_T:
        T = args.long_T
    case = synth.make_prefill_case(T, H, d, W, k, ns, zipf=True, scale=1.0, seed=0, device=dev)
    O = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(T, W + k, dtype=torch.int32, device=dev)
    Os = [torch.empty_like(O) for _ in range(ns)]
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_BF16, 1, ch, T, H, d, W, k), dev)

    def step():
        for c0 in range(0, T, ch):
            c1 = min(T, c0 + ch)
            hs2.hs2_full_attn_select(case.Q[c0:c1], case.K[:c1], case.V[:c1], O[c0:c1], idx[c0:c1], ws,
                                     window=W, topk=k, q_start=c0)
        for l in range(ns):
            hs2.hs2_sparse_attn_prefill(case.Q_sparse[l], case.K, case.V, idx, Os[l])

    step()
    torch.cuda.synchronize()
    hs2.hs2_profile_enable(True)
    t = timed_steps(step, 2, lambda: None, stream)
    prof = per_kernel(hs2.hs2_profile_collect())
    hs2.hs2_profile_enable(False)
    st = hs2.hs2_device_status()
    if st != 0:
        raise RuntimeError(f"device status {hs2.STATUS.get(st)} in the 256k prefill")
    ms = statistics.median(t)
    full_fl, sp1, sp_fl, sig_fl = prefill_flops(T, H, d, W, k, ns)
    sel_ms = sum(prof.get(n, {"total_ms": 0.0})["total_ms"] for n in
                 ("fa_fwd_kernel", "select_sigma_kernel", "topk_select_kernel")) / 2
    sel_ach = full_fl / (sel_ms * 1e-3) / 1e12
    sp_ms = sum(v["total_ms"] for n, v in prof.items() if "sparse" in n) / 2
    res = {"workload": f"prefill T={T} H={H} d={d} in {ch}-query chunks over the causal prefix, Zipf key norms, "
                       f"window {W} + top-{k}, {ns} sparse layers",
           "step_ms": ms, "tflops": (full_fl + sp_fl) / (ms * 1e-3) / 1e12,
           "select_call_ms": sel_ms, "select_call_tflops": sel_ach,
           "select_call_frac": sel_ach / peaks["bf16_tflops"], "algorithmic_flops_full": full_fl,
           "executed_extra_flops_sigma_pass": sig_fl, "sparse_ms": sp_ms,
           "sparse_tflops": sp_fl / (sp_ms * 1e-3) / 1e12 if sp_ms > 0 else None,
           "peak": peaks["bf16_tflops"], "peak_source": f"{peak_src} bf16_tflops",
           "l2": "inputs larger than L2 (Q 2.15 GB, sigma 8.6 GB per chunk)", "kernels": prof}
    del case, O, idx, Os, ws
    return res


def bench_swa(hs2, case, flush, stream, peaks, window=128):
    """A self-decoder sliding-window layer at the prefill head shape (the
    step's Q, K, V; window 128, 64-dim partial RoPE)."""
    T, H, d = case.Q.shape
    O = torch.empty_like(case.Q)
    ws = hs2.workspace(hs2.hs2_swa_attn_prefill_workspace(T, T, H, d), case.Q.device)

    def call():
        hs2.hs2_swa_attn_prefill(case.Q, case.K, case.V, O, ws, window=window)

    warm_up(call)
    hs2.hs2_profile_enable(True)
    t = timed_steps(call, 5, flush, stream)
    prof = per_kernel(hs2.hs2_profile_collect())
    hs2.hs2_profile_enable(False)
    ms = statistics.median(t)
    pairs = sum(min(p + 1, window) for p in range(T))
    fl = 4.0 * d * H * pairs
    return {"workload": f"sliding-window attention T={T} H={H} d={d}, window {window}, 64-dim partial RoPE",
            "ms": ms, "tflops": fl / (ms * 1e-3) / 1e12, "algorithmic_flops": fl,
            "kernels": {k: v["avg_ms"] for k, v in prof.items()}}


def bench_tiny(hs2, dev, stream, flush, args):
    """The tiny single-sequence case (T = 1024, 8 heads, d = 128, window 128 +
    top-256, 1 sparse layer): launch-bound, reported only."""
    import synth
    c = synth.CONFIGS[1]
    T, H, d, W, k = c["T"], c["H"], c["d"], c["window"], c["topk"]
    case = synth.make_prefill_case(T, H, d, W, k, c["n_sparse"], n_needles=c["n_needles"], seed=0, device=dev)
    O = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(T, W + k, dtype=torch.int32, device=dev)
    Os = torch.empty_like(O)
    ws = hs2.workspace(hs2.hs2_full_attn_select_workspace(hs2.KV_BF16, 1, T, T, H, d, W, k), dev)

    def step():
        hs2.hs2_full_attn_select(case.Q, case.K, case.V, O, idx, ws, window=W, topk=k)
        hs2.hs2_sparse_attn_prefill(case.Q_sparse[0], case.K, case.V, idx, Os)

    warm_up(step)
    hs2.hs2_profile_enable(True)
    t = timed_steps(step, max(5, args.steps), flush, stream)
    prof = per_kernel(hs2.hs2_profile_collect())
    hs2.hs2_profile_enable(False)
    full_fl, sp1, sp_fl, _ = prefill_flops(T, H, d, W, k, 1)
    ms = statistics.median(t)
    return {"workload": f"prefill T={T} H={H} d={d}, window {W} + top-{k}, 1 sparse layer, 4 needles",
            "step_ms": ms, "tflops": (full_fl + sp_fl) / (ms * 1e-3) / 1e12,
            "bound": "launch (4 kernels of a few microseconds each)", "kernels": prof}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-bridge", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-long", action="store_true", help="skip the 256k chunked prefill")
    ap.add_argument("--no-blocks", action="store_true", help="skip the block-level selection call")
    ap.add_argument("--bridge-rows", type=int, default=None,
                    help="override the bridged workload's rows, 4 sequences of rows/4 tokens (small profiling cases)")
    ap.add_argument("--long-T", type=int, default=None, help="override the chunked prefill length (small profiling cases)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=48)
    ap.add_argument("--T", type=int, default=None, help="override the prefill length (small profiling cases)")
    ap.add_argument("--decode-N", type=int, default=None, help="override the decode context (small profiling cases)")
    ap.add_argument("--only-decode", action="store_true", help="run the decode measurement only")
    ap.add_argument("--decode-B", type=int, default=None, help="override the decode batch (small profiling cases)")
    ap.add_argument("--sharded-nccl", action="store_true",
                    help="run only the context-sharded 1M decode over NCCL (also as a single rank)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    if args.decode_N:
        DECODE["N"] = args.decode_N
    if args.decode_B:
        DECODE["B"] = args.decode_B
    if args.bridge_rows:
        BRIDGE["R"] = args.bridge_rows
    if args.T:
        WORKLOAD["T"] = args.T
        WORKLOAD["n_needles"] = min(WORKLOAD["n_needles"], max(0, args.T // 512))

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return
    dist = world > 1 or args.sharded_nccl
    if dist:
        import datetime
        local = int(os.environ.get("LOCAL_RANK", "0"))
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")   # a single rank started without torchrun
        os.environ.setdefault("MASTER_PORT", "29533")
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", rank=rank, world_size=world,
                                             timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    try:
        run_ours(args, rank, world, dist)
    finally:
        if dist:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
