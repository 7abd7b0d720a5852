"""Context-sharded decode (token_level_kv_b200.sharded) on one GPU: every shard
of the context runs in this process, and the exchanges between the library's
per-shard calls are done here with torch (stack for the all-gather, a sum for
the all-reduce) in place of NCCL.  The merged full-attention output, the index
row and the sparse layers' outputs are checked against the fp64 oracle on the
whole cache, under the same rules as the single-GPU decode."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity import TOL_FP8, check_idx_row, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hs2():
    import token_level_kv_b200 as m
    return m


class LocalExchange:
    """Every shard in this process: the all-gather stacks the shards' tensors,
    the all-reduce writes their sum into each."""

    def all_gather(self, local):
        return torch.stack(local)

    def all_reduce_sum(self, local):
        total = torch.stack(local).sum(0)
        for t in local:
            t.copy_(total)


def _run(hs2, case, R, bounds=None, W=128, k=1024):
    from token_level_kv_b200 import sharded
    B, N, H, d = case.B, case.N, case.H, case.d
    sd = sharded.ShardedDecode(kv_len=N, n_shards=R, shards=list(range(R)), batch=B, Hq=H, d=d, window=W, topk=k,
                               exchange=LocalExchange(), bounds=bounds)
    caches = []
    for off, n in sd.bounds:
        caches.append(tuple(t[:, off:off + n].contiguous().cuda() for t in (case.Kc, case.Vc, case.ks, case.vs)))
    O, idx, outs = sd.step(case.Q.cuda(), caches, [q.cuda() for q in case.Q_sparse])
    assert hs2.hs2_device_status() == 0
    return O.cpu(), idx.cpu(), [o.cpu() for o in outs]


def _check(case, O, idx, outs, W=128, k=1024):
    B, N = case.B, case.N
    ref = oracle.decode_select(case.Q, case.Kc, case.Vc, case.ks, case.vs, range(B), N, W, k)
    for b in range(B):
        ok, _, msg = check_idx_row(idx[b].numpy(), ref[b], W, k)
        assert ok, msg
        assert max_abs(O[b].float().numpy(), ref[b].O) <= TOL_FP8
    gidx = idx.numpy()                      # staged: the sparse layers read the index the step produced
    for Qs, Os in zip(case.Q_sparse, outs):
        sref = oracle.sparse_attn_decode(Qs, case.Kc, case.Vc, case.ks, case.vs, gidx, range(B))
        for b in range(B):
            assert max_abs(Os[b].float().numpy(), sref[b]) <= TOL_FP8


@pytest.mark.parametrize("B,N,H,d,R", [(2, 5000, 16, 256, 2), (1, 20000, 16, 256, 3), (3, 9000, 8, 128, 4),
                                       (2, 900, 16, 256, 2)])
def test_sharded_decode_matches_oracle(hs2, B, N, H, d, R):
    """Two to four shards; 900 keys: fewer candidates than the top-k, all taken."""
    case = synth.make_decode_case(B, N, H, d, 128, 1024, n_sparse=2, seed=30 + R)
    O, idx, outs = _run(hs2, case, R)
    _check(case, O, idx, outs)


def test_sharded_decode_uneven_shards(hs2):
    """Shards of unequal length; the last one lies inside the window (no
    candidates), the first holds fewer candidates than the top-k."""
    B, N = 2, 6000
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=1, seed=34)
    bounds = [(0, 700), (700, 5200), (5900, 100)]
    O, idx, outs = _run(hs2, case, 3, bounds=bounds)
    _check(case, O, idx, outs)


def test_sharded_decode_ties_go_to_smaller_positions(hs2):
    """Every key identical: the selection is positions 0..1023 exactly, across
    the shard boundaries (the shards' lists merge in position order)."""
    B, N = 2, 6000
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=0, seed=35)
    case.Kc[:] = case.Kc[:, :1]
    case.ks[:] = case.ks[:, :1]
    _, idx, _ = _run(hs2, case, 3, bounds=[(0, 640), (640, 2000), (2640, 3360)])
    for b in range(B):
        assert idx[b, 128:].tolist() == list(range(1024))
        assert idx[b, :128].tolist() == list(range(N - 128, N))


@pytest.mark.parametrize("B,N", [(1, 200000), (2, 300000)])
def test_sharded_decode_long_shards(hs2, B, N):
    """Shards of 100,000 candidates (each shard's top-k over several slices and
    a merge) and of 150,000 (the radix select over the GPU, written as the
    shard's list), then the merge across shards."""
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=1, seed=36)
    O, idx, outs = _run(hs2, case, 2)
    _check(case, O, idx, outs)


def test_shard_calls_reject_bad_arguments(hs2):
    ml = torch.zeros(2, 1, 16, device="cuda")
    O32 = torch.zeros(1, 16, 256, device="cuda")
    with pytest.raises(hs2.Hs2Error):
        hs2.hs2_partial_merge(ml.view(1, 2, 1, 16), 1, O32, torch.zeros(1, 16, 2, device="cuda"))
    cand = torch.zeros(65, hs2.candidates_numel(1, 16), dtype=torch.int32, device="cuda")
    with pytest.raises(hs2.Hs2Error):                  # at most 64 shards
        hs2.hs2_decode_merge_candidates(cand, torch.empty(1, 144, dtype=torch.int32, device="cuda"), kv_len=5000,
                                        window=128, topk=16)
    assert hs2.hs2_device_status() == 0


def test_sharded_decode_ties_inside_the_cut(hs2):
    """Two shards of 150,000 candidates each (the radix select writing the
    shards' lists), strong keys and a run of exactly tied keys around the cut:
    the merged selection is the strong keys plus the first tied keys in
    position order across the shard boundary's lists."""
    from hs2_cases import plant_tie_keys
    B, N, k = 1, 300000, 1024
    case = synth.make_decode_case(B, N, 16, 256, 128, k, n_sparse=0, seed=37)
    planted = plant_tie_keys(case, n_strong=300, tie_every=400)
    _, idx, _ = _run(hs2, case, 2)
    strong, ties = planted[0]
    want = np.sort(np.concatenate([strong, ties[:k - len(strong)]]))
    assert ties[k - len(strong) - 1] > 150000 and len(ties) > k - len(strong)   # taken ties in both shards, cut inside
    assert np.array_equal(idx[0, 128:].numpy(), want)
