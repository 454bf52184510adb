"""Pins of the oracle's activation-quantized linear (per-token INT8
activations, integer dot products per weight group; auto-round-lib README:
INT8 compute with dynamic activation quantization): the per-token scale
against an exact rational, the quantization error bound, and the reduction to
the weight-only linear when the activations already lie on their INT8 grid."""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest

import synth


def test_activation_scale_and_error_bound(orc):
    M, K = 12, 384
    x = synth.activations(5, M, K, channel_count=4, channel_mult=10.0)
    x[3] = 0                                              # an all-zero token
    xq, sx = orc.quant_act_int8(x)
    xv = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for m in range(M):
        amax = np.abs(xv[m]).max()
        if amax == 0:
            assert sx[m] == 0 and not xq[m].any()
            continue
        ulp = Fraction(float(np.spacing(np.float32(sx[m]))))
        assert abs(Fraction(float(sx[m])) - Fraction(amax) / 127) <= ulp / 2
        assert np.abs(xq[m].astype(np.int64)).max() == 127
        err = np.abs(xv[m] - xq[m].astype(np.float64) * float(sx[m]))
        assert np.all(err <= 0.5 * float(sx[m]) * (1 + 1e-12))


@pytest.mark.parametrize("fmt", ["int8_sym", "int4_sym"])
def test_grid_activations_reduce_to_weight_only_linear(orc, fmt):
    """x = integers * 2^-e with every row reaching 127 * 2^-e: the INT8
    activations are exact, so (one weight group per row) the result equals the
    weight-only linear's fp64 sum exactly."""
    N, K = 40, 256
    W = synth.weight(8, N, K, sigma=0.02)
    codes, scales, _ = orc.quantize(fmt, W, K)
    rng = np.random.default_rng(4)
    M = 6
    ints = rng.integers(-127, 128, size=(M, K))
    ints[:, 0] = 127
    e = rng.integers(3, 9, size=(M, 1))
    x = synth.f64_to_bf16_bits(ints * np.ldexp(1.0, -e))
    b = synth.bias(8, N)
    y8, y8_64 = orc.linear_a8(fmt, codes, scales, N, K, K, x, b)
    dq = orc.dequant(fmt, codes, scales, None, N, K, K)
    y, y64 = orc.linear(x, dq, b)
    assert np.array_equal(y8_64, y64) and np.array_equal(y8, y)


@pytest.mark.parametrize("G", [32, 128, 256])
def test_a8_full_equals_loop(orc, G):
    """The matmul form of the activation-quantized linear gives the same fp64
    numbers as the oracle's loop (exact integer group sums, the same scaling
    and accumulation order), hence the same bf16 outputs; with and without
    bias, on outlier channels."""
    N, K, M = 48, 512, 7
    W = synth.weight(9, N, K, sigma=0.02, outlier_count=20, outlier_mult=20.0)
    codes, scales, _ = orc.quantize("int8_sym", W, G)
    x = synth.activations(10, M, K, channel_count=5, channel_mult=10.0)
    b = synth.bias(9, N)
    for bias in (b, None):
        y, y64 = orc.linear_a8("int8_sym", codes, scales, N, K, G, x, bias)
        yf, yf64 = orc.linear_a8_full(codes, scales, N, K, G, x, bias)
        assert np.array_equal(yf64, y64) and np.array_equal(yf, y)


def test_a8_full_integer_case(orc):
    """Unit scales and activations on the INT8 grid with s_x = 1 (row max 127):
    y is the integer matmul of the codes."""
    N, K, M, G = 24, 256, 5, 64
    rng = np.random.default_rng(11)
    q = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    scales = np.full((N, K // G), 0x3F80, np.uint16)
    xi = rng.integers(-127, 128, size=(M, K))
    xi[:, 3] = 127
    x = synth.f64_to_bf16_bits(xi.astype(np.float64))
    y, y64 = orc.linear_a8_full(q, scales, N, K, G, x, None)
    ref = (xi @ q.astype(np.int64).T).astype(np.float64)
    assert np.array_equal(y64, ref)


def test_a8_full_int4_equals_loop(orc):
    """The matmul form with INT4 codes (two's complement nibbles) equals the loop."""
    N, K, M, G = 32, 256, 5, 64
    W = synth.weight(12, N, K, sigma=0.02)
    codes, scales, _ = orc.quantize("int4_sym", W, G)
    x = synth.activations(13, M, K)
    y, y64 = orc.linear_a8("int4_sym", codes, scales, N, K, G, x, None)
    yf, yf64 = orc.linear_a8_full(codes, scales, N, K, G, x, None)
    assert np.array_equal(yf64, y64) and np.array_equal(yf, y)
