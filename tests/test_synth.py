"""The seeded input generator (CPU only)."""
import math

import torch

import synth


def _ref_bits(seed, stream, i):
    M = (1 << 64) - 1

    def mix(z):
        z &= M
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
        return z ^ (z >> 31)
    key = mix(seed * 0xD1B54A32D192ED03 + stream)
    return mix(key + (i + 1) * 0x9E3779B97F4A7C15)


def test_bits_match_plain_integer_definition():
    got = synth.bits(7, 3, 1000, 64)
    for j in range(64):
        assert (int(got[j]) & ((1 << 64) - 1)) == _ref_bits(7, 3, 1000 + j)


def test_normal_moments_and_determinism():
    z = synth.normal(0, 1, 1 << 20)
    assert abs(float(z.mean())) < 5e-3
    assert abs(float(z.std()) - 1.0) < 5e-3
    assert torch.equal(z[1234:1300], synth.normal(0, 1, 66, start=1234))


def test_zipf_norms_amplify_36_keys():
    n = synth.zipf_key_norms(5000, 0)
    assert int((n > 1).sum()) == 35          # rank 36 gives exactly 1.0
    assert float(n.max()) == 6.0 and float(n.min()) == 1.0


def test_fp8_rows_reach_448_and_scales_are_amax_over_448():
    codes, sc = synth.fp8_rows_from_normal(0, 2, 2, 50, 64)
    v = codes.view(torch.float8_e4m3fn).to(torch.float32)
    assert torch.all(v.abs().amax(-1) == 448.0)
    x = synth.normal(0, 2, 2 * 50 * 64).to(torch.bfloat16).float().view(2, 50, 64)
    assert torch.allclose(sc, x.abs().amax(-1) / 448.0, rtol=0, atol=0)


def test_needle_rows_have_the_planted_mean_logit():
    case = synth.make_prefill_case(512, 8, 64, 32, 16, n_sparse=0, n_needles=3)
    for p, i in case.needles:
        assert i >= p + 32
        s = (case.Q[i].double() @ case.K[p].double()) / math.sqrt(64)
        assert abs(float(s.mean()) - 8.0) < 0.1      # bf16 rounding of K[p]
