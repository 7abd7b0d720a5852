"""The context-sharded decode's orchestration (token_level_kv_b200.sharded)
over world-size-2 gloo ranks on the CPU: each rank holds one shard of every
sequence's FP8 cache and runs the per-shard steps (CPU stand-ins written from
the library's contracts, tests/sharded_cpu_ops.py) with the real exchanges
(all-gather, all-reduce) between them.  Every rank's index row and outputs
must match the fp64 oracle on the whole cache."""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, N, bounds, out):
    sys.path[:0] = [ROOT, HERE]
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from parity import TOL_FP8, check_idx_row, max_abs
    from sharded_cpu_ops import CpuOps
    from token_level_kv_b200 import sharded

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        B, H, d, W, k = 2, 16, 256, 128, 1024
        case = synth.make_decode_case(B, N, H, d, W, k, n_sparse=1, seed=40)
        sd = sharded.ShardedDecode(kv_len=N, n_shards=world, shards=[rank], batch=B, Hq=H, d=d, window=W, topk=k,
                                   exchange=sharded.GroupExchange(), ops=CpuOps, device="cpu", bounds=bounds)
        off, n = sd.bounds[rank]
        cache = tuple(t[:, off:off + n].contiguous() for t in (case.Kc, case.Vc, case.ks, case.vs))
        O, idx, outs = sd.step(case.Q, [cache], case.Q_sparse)
        ref = oracle.decode_select(case.Q, case.Kc, case.Vc, case.ks, case.vs, range(B), N, W, k)
        sref = oracle.sparse_attn_decode(case.Q_sparse[0], case.Kc, case.Vc, case.ks, case.vs, idx.numpy(),
                                         range(B))
        msgs = []
        for b in range(B):
            ok, _, msg = check_idx_row(idx[b].numpy(), ref[b], W, k)
            if not ok:
                msgs.append(msg)
            if max_abs(O[b].float().numpy(), ref[b].O) > TOL_FP8:
                msgs.append(f"full-attention output of sequence {b}")
            if max_abs(outs[0][b].float().numpy(), sref[b]) > TOL_FP8:
                msgs.append(f"sparse output of sequence {b}")
        out[rank] = (msgs, idx.numpy().tobytes(), n)
    finally:
        dist.destroy_process_group()


def _run(N, bounds=None, world=2):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), N, bounds, out), nprocs=world, start_method="spawn")
    for r in range(world):
        assert out[r][0] == [], out[r][0]
    # every rank ends the step with the same index row
    assert all(out[r][1] == out[0][1] for r in range(world))
    return [out[r][2] for r in range(world)]


def test_two_ranks_equal_shards():
    lens = _run(3000)
    assert lens == [1472, 1528]


def test_two_ranks_second_shard_inside_the_window():
    """Rank 1 holds only the last 100 positions: no candidates of its own."""
    lens = _run(2500, bounds=[(0, 2400), (2400, 100)])
    assert lens == [2400, 100]


def test_shard_bounds_tile_the_context():
    sys.path.insert(0, ROOT)
    from token_level_kv_b200.sharded import shard_bounds
    for kv, R in [(1 << 20, 8), (3000, 2), (1000, 3), (64 * 7 + 5, 7), (100, 3)]:
        b = shard_bounds(kv, R)
        assert b[0][0] == 0 and sum(n for _, n in b) == kv
        assert all(b[i][0] + b[i][1] == b[i + 1][0] for i in range(R - 1))
        assert all(n > 0 for _, n in b) and (kv < 64 * R or all(o % 64 == 0 for o, _ in b))
    assert np.array_equal(shard_bounds(1 << 20, 4), [(q << 18, 1 << 18) for q in range(4)])


def test_shard_bounds_refuse_more_shards_than_positions():
    import pytest
    sys.path.insert(0, ROOT)
    from token_level_kv_b200.sharded import shard_bounds
    with pytest.raises(ValueError):
        shard_bounds(3, 4)
    with pytest.raises(ValueError):
        shard_bounds(100, 0)
    assert shard_bounds(5, 5) == [(i, 1) for i in range(5)]
