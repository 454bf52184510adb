"""The seeded input generator: determinism, the published SplitMix64 constants,
distribution sanity and the outlier recipes."""
from __future__ import annotations

import numpy as np
from scipy import stats

import synth
import synth.workloads as W


def test_splitmix64_reference_values():
    """SplitMix64 seeded with 0 (Vigna's published generator): first outputs."""
    assert synth.splitmix64(0, 0) == 0xE220A8397B1DCDAF
    assert synth.splitmix64(0, 1) == 0x6E789E6AA1B965F4
    assert synth.splitmix64(0, 2) == 0x06C45D188009454F


def test_streams_are_deterministic_and_distinct():
    a = synth.normal_stream(1, 1, 0, 1000)
    b = synth.normal_stream(1, 1, 0, 1000)
    c = synth.normal_stream(1, 2, 0, 1000)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    # any window of the stream equals the same slice of a longer draw
    assert np.array_equal(synth.normal_stream(1, 1, 500, 100), a[500:600])


def test_distributions():
    u = synth.uniform_stream(0, 9, 0, 200000)
    assert 0 < u.min() and u.max() < 1
    assert stats.kstest(u, "uniform").pvalue > 1e-3
    z = synth.normal_stream(0, 9, 0, 200000)
    assert stats.kstest(z, "norm").pvalue > 1e-3
    t = synth.student5_stream(0, 9, 0, 100000)
    assert stats.kstest(t, stats.t(5).cdf).pvalue > 1e-3


def test_weight_outliers_and_channels():
    w = synth.weight(1, 64, 128, sigma=0.02, outlier_count=80, outlier_mult=20.0)
    base = synth.weight(1, 64, 128, sigma=0.02)
    ratio = w / np.where(base == 0, 1, base)
    assert np.sum(np.isclose(ratio, 20.0, rtol=1e-6)) == 80
    pos = synth.distinct_positions(1, 4, 64 * 128, 80)
    assert len(set(pos.tolist())) == 80
    x = synth.activations(4, 8, 256, channel_count=3, channel_mult=10.0)
    x0 = synth.activations(4, 8, 256)
    assert not np.array_equal(x, x0)
    cols = np.where(np.any(x != x0, axis=0))[0]
    assert len(cols) == 3


def test_workload_recipes():
    assert W.DECODE.w_outlier_count == 16777
    assert W.PREFILL.x_channel_count == 82
    assert W.algorithmic_bytes(W.PR1, 4) == 76288
    assert W.algorithmic_bytes(W.DECODE, 1) == 8716288 + 16384
    assert W.algorithmic_bytes(W.NVFP4, 1) == 132120580 + 73728
    # MXFP4: codes N*K/2 + one E8M0 byte per 32; FP8: N*K + fp32 scale per group
    assert W.algorithmic_bytes(W.MXFP4, 1) == 28672 * 8192 // 2 + 28672 * 256 + 73728
    assert W.algorithmic_bytes(W.FP8, 1) == 8192 * 8192 + 4 * 8192 * 64 + 2 * 8192 + 2 * 8192
    assert W.packed_bytes("int2_sym", 256, 512, 64) == 256 * 128 + 2 * 256 * 8
    assert len({w.seed for w in W.ALL}) == len(W.ALL)       # one stream per workload
    x1 = W.make_x(W.DECODE, 1)
    x16 = W.make_x(W.DECODE, 16)
    assert np.array_equal(x1[0], x16[0])
