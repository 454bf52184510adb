"""Pins of the oracle's LoRA merge into an INT8 weight (piper-kernels README:
weight.addmm_(mat1, mat2, alpha) computes beta*weight + alpha*(mat1 @ mat2)
and requantizes with the unchanged scales; with a rounding seed it picks one
of the two adjacent codes with probability proportional to distance):
closed forms where the update is a whole number of scale steps, numpy's
round-half-even, the stochastic rule against an independent SplitMix64
(the input generator's), and its statistics."""
from __future__ import annotations

import numpy as np

import synth


def _case(orc, N=64, K=256, seed=3):
    W = synth.weight(seed, N, K, sigma=0.02)
    codes, scales, _ = orc.quantize("int8_sym", W, K)     # one group (scale) per row
    return codes, scales


def _bits(v):
    return synth.f64_to_bf16_bits(np.asarray(v, dtype=np.float64))


def test_identity_and_whole_steps(orc):
    codes, scales = _case(orc)
    N, K = codes.shape
    z1, z2 = _bits(np.zeros((N, 1))), _bits(np.zeros((1, K)))
    for seed in (None, 5):
        assert np.array_equal(orc.addmm_requant_int8(codes, scales, K, z1, z2, 1.0, 1.0, seed),
                              codes)
    # mat1[n] = the row's scale, mat2[k] = integers d: the update is d steps exactly
    d = np.random.default_rng(1).integers(-3, 4, size=(1, K))
    m1 = scales.reshape(N, 1).copy()                      # bf16 bits of s_n
    want = np.clip(codes.astype(np.int64) + d, -127, 127)
    for seed in (None, 9):
        got = orc.addmm_requant_int8(codes, scales, K, m1, _bits(d), 1.0, 1.0, seed)
        assert np.array_equal(got.astype(np.int64), want)
    # saturation
    big = orc.addmm_requant_int8(codes, scales, K, m1, _bits(np.full((1, K), 300.0)), 1.0, 1.0)
    assert np.all(big == 127)


def test_beta_halves_with_ties_to_even(orc):
    codes, scales = _case(orc, seed=4)
    N, K = codes.shape
    z1, z2 = _bits(np.zeros((N, 1))), _bits(np.zeros((1, K)))
    got = orc.addmm_requant_int8(codes, scales, K, z1, z2, 1.0, 0.5)
    assert np.array_equal(got.astype(np.int64), np.rint(codes.astype(np.float64) / 2))


def test_stochastic_rule_against_independent_splitmix(orc):
    codes, scales = _case(orc, N=32, K=512, seed=6)
    N, K = codes.shape
    rng = np.random.default_rng(2)
    frac = rng.integers(1, 8, size=(1, K)) / 8.0           # exact in bf16
    m1 = scales.reshape(N, 1).copy()
    seed = 0x1234
    got = orc.addmm_requant_int8(codes, scales, K, m1, _bits(frac), 1.0, 1.0, seed)
    idx = np.arange(N * K, dtype=np.uint64)
    u = np.array([synth.splitmix64(seed, int(i)) >> 11 for i in idx], dtype=np.float64) * 2.0 ** -53
    up = (u.reshape(N, K) < np.broadcast_to(frac, (N, K))).astype(np.int64)
    want = np.clip(codes.astype(np.int64) + up, -127, 127)
    assert np.array_equal(got.astype(np.int64), want)
    # another seed gives another (valid) choice
    other = orc.addmm_requant_int8(codes, scales, K, m1, _bits(frac), 1.0, 1.0, seed + 1)
    assert not np.array_equal(other, got)
    assert np.all(np.isin(other.astype(np.int64) - codes.astype(np.int64), [0, 1]) |
                  (codes == 127))


def test_stochastic_rounding_is_unbiased(orc):
    codes, scales = _case(orc, N=128, K=512, seed=7)
    N, K = codes.shape
    m1 = scales.reshape(N, 1).copy()
    got = orc.addmm_requant_int8(codes, scales, K, m1, _bits(np.full((1, K), 0.25)), 1.0, 1.0,
                                 seed=77)
    inc = (got.astype(np.int64) - codes.astype(np.int64))[codes < 127]
    assert set(np.unique(inc)) <= {0, 1}
    assert abs(inc.mean() - 0.25) < 0.01
