"""Pins of the oracle's linear: exact rational brute force on tiny K, an
integer-valued special case per format that reduces to an integer matmul, and
the sampled path against the full one."""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0,
                 -4.0, -6.0])


def _pack_nibbles(vals):
    """u8 [N, K] values 0..15 -> canonical u8 [N, K/2], element 2i in the low nibble."""
    v = np.asarray(vals, dtype=np.uint8)
    return (v[:, 0::2] | (v[:, 1::2] << 4)).astype(np.uint8)


def _bf16_exact_rne(v: Fraction) -> Fraction:
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = 0
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    q = Fraction(2) ** (e - 7)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * q


@pytest.mark.parametrize("K", [1, 2, 7, 16, 32])
def test_linear_matches_exact_rational(orc, K):
    M, N = 3, 5
    rng = np.random.default_rng(K)
    x = synth.f64_to_bf16_bits(rng.standard_normal((M, K)))
    dq = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    b = synth.f64_to_bf16_bits(rng.standard_normal(N) * 0.01)
    y, y64 = orc.linear(x, dq, b)
    xf = oracle.bits_to_f32(x)
    bf = oracle.bits_to_f32(b)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xf[m, k])) * Fraction(float(dq[n, k])) for k in range(K))
            exact += Fraction(float(bf[n]))
            absum = sum(abs(float(xf[m, k]) * float(dq[n, k])) for k in range(K)) + abs(float(bf[n]))
            assert abs(Fraction(float(y64[m, n])) - exact) <= Fraction((K + 1) * 2.0 ** -52 * absum)
            want = _bf16_exact_rne(exact)
            got = Fraction(float(oracle.bits_to_f32(np.array([y[m, n]], np.uint16))[0]))
            # equal unless the exact value sits within the fp64 error of a bf16 tie
            if got != want:
                tie_dist = abs(exact - (got + want) / 2)
                assert tie_dist <= Fraction((K + 1) * 2.0 ** -52 * absum)


def _int_case(fmt, N, K, G, rng):
    """Canonical data whose dequantized values are small integers (or halves)."""
    if fmt == "int4_sym":
        v = rng.integers(-8, 8, size=(N, K))
        codes = _pack_nibbles(v & 15)
        scales = np.full((N, K // G), 0x3F80, np.uint16)   # 1.0
        return codes, scales, None, v.astype(np.float64)
    if fmt == "int2_sym":
        v = rng.integers(-2, 2, size=(N, K))          # every 2-bit code, -2 included
        c = (v & 3).reshape(N, K // 4, 4)
        codes = (c[..., 0] | (c[..., 1] << 2) | (c[..., 2] << 4) | (c[..., 3] << 6)).astype(np.uint8)
        scales = np.full((N, K // G), 0x3F80, np.uint16)
        return codes, scales, None, v.astype(np.float64)
    if fmt == "int3_sym":
        v = rng.integers(-4, 4, size=(N, K))          # every 3-bit code, -4 included
        bits = np.stack([(v >> b) & 1 for b in range(3)], axis=-1).reshape(N, -1)
        codes = np.packbits(bits.astype(np.uint8), axis=1, bitorder="little")
        scales = np.full((N, K // G), 0x3F80, np.uint16)
        return codes, scales, None, v.astype(np.float64)
    if fmt == "int4_asym":
        q = rng.integers(0, 16, size=(N, K))
        z = rng.integers(0, 16, size=(N, K // G))
        codes = _pack_nibbles(q)
        scales = np.full((N, K // G), 0x3F80, np.uint16)
        return codes, scales, z.astype(np.uint8), (q - np.repeat(z, G, axis=1)).astype(np.float64)
    if fmt == "int8_sym":
        v = rng.integers(-128, 128, size=(N, K))
        scales = np.full((N, K // G), 0x3F80, np.uint16)
        return v.astype(np.int8), scales, None, v.astype(np.float64)
    if fmt == "cb4":
        idx = rng.integers(0, 16, size=(N, K))
        cent = (np.arange(16) - 8).astype(np.float32) * 3   # integer centroids
        norms = np.full((N,), 0x3F80, np.uint16)
        return _pack_nibbles(idx), norms, cent, cent.astype(np.float64)[idx]
    if fmt == "nvfp4":
        q = rng.integers(0, 16, size=(N, K))
        q[q == 8] = 0
        bs = np.full((N, K // 16), 0x38, np.uint8)         # E4M3 1.0
        ts = np.array([1.0], np.float32)
        return _pack_nibbles(q), bs, ts, E2M1[q]
    if fmt == "mxfp4":
        q = rng.integers(0, 16, size=(N, K))
        q[q == 8] = 0
        bs = np.full((N, K // 32), 127, np.uint8)          # E8M0 1.0
        return _pack_nibbles(q), bs, None, E2M1[q]
    if fmt == "fp8_e4m3":
        # E4M3 codes of the integers -16..16 (exact): 2^e (1 + m/8)
        v = rng.integers(-16, 17, size=(N, K))
        a = np.abs(v)
        e = np.floor(np.log2(np.maximum(a, 1))).astype(np.int64)
        m = (a * 8 // (1 << e)) - 8
        code = np.where(a == 0, 0, ((e + 7) << 3) | m) | np.where(v < 0, 0x80, 0)
        scales = np.ones((N, K // G), np.float32)
        return code.astype(np.uint8), scales, None, v.astype(np.float64)
    if fmt == "fp8_e5m2":
        # E5M2 codes of the integers -8..8 (exact): 2^e (1 + m/4)
        v = rng.integers(-8, 9, size=(N, K))
        a = np.abs(v)
        e = np.floor(np.log2(np.maximum(a, 1))).astype(np.int64)
        m = (a * 4 // (1 << e)) - 4
        code = np.where(a == 0, 0, ((e + 15) << 2) | m) | np.where(v < 0, 0x80, 0)
        scales = np.ones((N, K // G), np.float32)
        return code.astype(np.uint8), scales, None, v.astype(np.float64)
    raise ValueError(fmt)


@pytest.mark.parametrize("fmt,G", [("int4_sym", 64), ("int4_asym", 32), ("int8_sym", 128),
                                   ("cb4", 0), ("nvfp4", 16), ("mxfp4", 32), ("fp8_e4m3", 64),
                                   ("fp8_e5m2", 32), ("int2_sym", 64), ("int3_sym", 32)])
def test_integer_special_case(orc, fmt, G):
    """Integer X, unit scales: every partial sum is exact, so y equals an
    integer matmul done by numpy -- pins layout, nibble order and orientation."""
    M, N, K = 5, 24, 256
    rng = np.random.default_rng(sum(map(ord, fmt)))
    codes, scales, aux, wval = _int_case(fmt, N, K, G, rng)
    xi = rng.integers(-4, 5, size=(M, K))
    x = synth.f64_to_bf16_bits(xi.astype(np.float64))
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    assert np.array_equal(dq.astype(np.float64), wval)
    y, y64 = orc.linear(x, dq, None)
    ref = xi.astype(np.float64) @ wval.T
    assert np.array_equal(y64, ref)
    assert np.array_equal(y, synth.f64_to_bf16_bits(ref))


@pytest.mark.parametrize("fmt,G", [("int4_sym", 64), ("int4_asym", 128), ("int8_sym", 256),
                                   ("cb4", 0), ("nvfp4", 16), ("mxfp4", 32), ("fp8_e4m3", 128),
                                   ("fp8_e5m2", 64), ("int2_sym", 32)])
def test_sampled_equals_full(orc, fmt, G):
    M, N, K = 6, 32, 512
    W = synth.weight(21, N, K, sigma=0.02)
    codes, scales, aux = orc.quantize(fmt, W, G)
    x = synth.activations(21, M, K)
    b = synth.bias(21, N)
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    y, y64 = orc.linear(x, dq, b)
    ms = np.repeat(np.arange(M), N)
    ns = np.tile(np.arange(N), M)
    ys, ys64 = orc.linear_sampled(fmt, codes, scales, aux, N, K, G, x, b, ms, ns)
    assert np.array_equal(ys.reshape(M, N), y)
    assert np.array_equal(ys64.reshape(M, N), y64)


def test_empty_batch(orc):
    dq = np.ones((4, 8), np.float32)
    x = np.zeros((0, 8), np.uint16)
    y, y64 = orc.linear(x, dq)
    assert y.shape == (0, 4)


@pytest.mark.parametrize("K", [1, 7, 32])
def test_linear_full_matches_exact_rational(orc, K):
    """The library-matmul product against exact rational sums (tiny K)."""
    M, N = 3, 5
    rng = np.random.default_rng(100 + K)
    x = synth.f64_to_bf16_bits(rng.standard_normal((M, K)))
    dq = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    b = synth.f64_to_bf16_bits(rng.standard_normal(N) * 0.01)
    y, y64 = orc.linear_full(x, dq, b)
    xf, bf = oracle.bits_to_f32(x), oracle.bits_to_f32(b)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xf[m, k])) * Fraction(float(dq[n, k])) for k in range(K))
            exact += Fraction(float(bf[n]))
            absum = sum(abs(float(xf[m, k]) * float(dq[n, k])) for k in range(K)) + abs(float(bf[n]))
            assert abs(Fraction(float(y64[m, n])) - exact) <= Fraction((K + 1) * 2.0 ** -52 * absum)
            want = _bf16_exact_rne(exact)
            got = Fraction(float(oracle.bits_to_f32(np.array([y[m, n]], np.uint16))[0]))
            if got != want:
                assert abs(exact - (got + want) / 2) <= Fraction((K + 1) * 2.0 ** -52 * absum)


@pytest.mark.parametrize("fmt,G", [("int4_asym", 128), ("nvfp4", 16), ("int8_sym", 256)])
def test_linear_full_equals_loop(orc, fmt, G):
    """The library-matmul product and the increasing-k loop agree: fp64 values
    within the summation-order bound, bf16 outputs identical (a difference
    needs an exact value within ~1e-13 of a bf16 rounding boundary).  A
    transposed weight, a dropped bias or another rounding would fail here.
    The chunking over rows is exercised by a chunk smaller than N."""
    M, N, K = 9, 272, 2048
    W = synth.weight(33, N, K, sigma=0.02, outlier_count=N * K // 1000, outlier_mult=20.0)
    codes, scales, aux = orc.quantize(fmt, W, G)
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    x = synth.activations(33, M, K)
    b = synth.bias(33, N)
    y, y64 = orc.linear(x, dq, b)
    yf, yf64 = orc.linear_full(x, dq, b, rows_per_chunk=96)
    absum = np.abs(oracle.bits_to_f32(x).astype(np.float64)) @ np.abs(dq.astype(np.float64)).T
    assert np.all(np.abs(yf64 - y64) <= 2 * (K + 1) * 2.0 ** -52 * (absum + 1.0))
    assert np.array_equal(yf, y)
    # no bias: the same product without the bias term
    y0, _ = orc.linear(x, dq, None)
    yf0, _ = orc.linear_full(x, dq, None)
    assert np.array_equal(yf0, y0)
    assert not np.array_equal(yf0, yf)


def test_linear_full_integer_case(orc):
    """Integer operands: the library product is exact and equals numpy's
    integer matmul bit for bit (orientation: y[m, n] = sum_k x[m, k] w[n, k])."""
    M, N, K = 5, 40, 256
    rng = np.random.default_rng(7)
    codes, scales, aux, wval = _int_case("int4_sym", N, K, 64, rng)
    xi = rng.integers(-4, 5, size=(M, K))
    x = synth.f64_to_bf16_bits(xi.astype(np.float64))
    dq = orc.dequant("int4_sym", codes, scales, aux, N, K, 64)
    y, y64 = orc.linear_full(x, dq, None)
    ref = (xi @ wval.astype(np.int64).T).astype(np.float64)
    assert np.array_equal(y64, ref)
    assert np.array_equal(y, synth.f64_to_bf16_bits(ref))
