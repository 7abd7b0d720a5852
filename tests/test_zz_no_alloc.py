"""hs2_sparse_attn_decode_static: the sparse decode for callers that cannot
allocate device memory (their device memory is reserved by their own pool, or
cudaMalloc's implicit synchronisation is not acceptable in their decode loop).
Its split scratch is the library's static device array, so it takes no
workspace.  Checked through the C ABI against hs2_sparse_attn_decode (which
takes a caller workspace) on two calls in a row, so that the second call also
shows that what the first left in the shared array does not leak into it.
Collected last on purpose: a run that stops at its first failure has already
run every other test."""
import numpy as np
import pytest
import torch

import synth
from parity import TOL_FP8, max_abs

pytestmark = pytest.mark.gpu


def _case(seed, B, N):
    case = synth.make_decode_case(B, N, 16, 256, 128, 1024, n_sparse=2, seed=seed, device="cuda")
    g = np.random.default_rng(seed)
    idx = np.full((B, 1152), -1, dtype=np.int32)
    for b in range(B):
        n = int(g.integers(1, 1153))
        idx[b, :n] = np.sort(g.choice(N, size=n, replace=False))
    return case, torch.from_numpy(idx).cuda()


def test_static_scratch_matches_workspace_path_two_calls_in_a_row():
    import token_level_kv_b200 as hs2
    B, N = 4, 3000                       # small batch: more splits than a cluster, so the scratch is used
    assert hs2.hs2_sparse_attn_decode_workspace(B, 1152, 16, 256) > 0
    cases = [_case(21, B, N), _case(22, B, N)]
    got = []
    for case, idx in cases:              # two calls in a row on the shared array
        O = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
        hs2.hs2_sparse_attn_decode_static(case.Q_sparse[0], case.Kc, case.Vc, case.ks, case.vs, idx, O)
        got.append(O)
    assert hs2.hs2_device_status() == 0
    for (case, idx), O in zip(cases, got):
        ref = torch.empty_like(O)
        ws = hs2.workspace(hs2.hs2_sparse_attn_decode_workspace(B, 1152, 16, 256))
        hs2.hs2_sparse_attn_decode(case.Q_sparse[0], case.Kc, case.Vc, case.ks, case.vs, idx, ref, ws)
        assert hs2.hs2_device_status() == 0
        assert max_abs(O.float().cpu().numpy(), ref.float().cpu().numpy()) <= TOL_FP8
        assert torch.equal(O, ref)       # same kernels, same splits: identical bits
