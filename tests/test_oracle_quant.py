"""Pins of the oracle's quantizers and dequantizer: closed-form round trips,
error bounds, code ranges and nearest-neighbour properties, checked against
numpy/scipy/torch rather than against the oracle."""
from __future__ import annotations

import os

import numpy as np
import pytest
from scipy import integrate, stats

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _nibbles(codes):
    """canonical u8 [N, K/2] -> u8 [N, K]: element 2i in the low nibble."""
    lo = codes & 0x0F
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def _signed_codes(fmt, codes):
    """canonical INT codes -> signed integers [N, K] (two's complement fields:
    2-bit element 4i+j at bits 2j of byte i, 4-bit element 2i+j at bits 4j)."""
    if fmt == "int8_sym":
        return codes.astype(np.int64)
    if fmt == "int4_sym":
        q = _nibbles(codes).astype(np.int64)
        return np.where(q > 7, q - 16, q)
    if fmt == "int3_sym":  # little-endian bit stream per row, element k at bits 3k..3k+2
        bits = np.unpackbits(codes.astype(np.uint8), axis=1, bitorder="little").astype(np.int64)
        bits = bits.reshape(codes.shape[0], -1, 3)
        q = bits[..., 0] | (bits[..., 1] << 1) | (bits[..., 2] << 2)
        return np.where(q > 3, q - 8, q)
    c = codes.astype(np.int64)
    q = np.stack([(c >> (2 * j)) & 3 for j in range(4)], axis=-1).reshape(codes.shape[0], -1)
    return np.where(q > 1, q - 4, q)


def _bf16(bits):
    return oracle.bits_to_f32(bits).astype(np.float64)


def _weights(N, K, seed=0, outliers=True):
    W = synth.weight(seed, N, K, sigma=0.02, outlier_count=(N * K) // 500 if outliers else 0,
                     outlier_mult=20.0)
    W[0, :] = 0.0                # an all-zero row (and groups)
    W[1, : K // 2] = 0.0
    return W


# --------------------------------------------------------------- symmetric INT
@pytest.mark.parametrize("fmt,qmax", [("int2_sym", 1), ("int3_sym", 3), ("int4_sym", 7),
                                      ("int8_sym", 127)])
@pytest.mark.parametrize("G", [32, 64, 128, 256])
def test_sym_properties(orc, fmt, qmax, G):
    N, K = 48, 512
    W = _weights(N, K, seed=G)
    codes, scales, _ = orc.quantize(fmt, W, G)
    q = _signed_codes(fmt, codes)
    s = _bf16(scales)
    assert np.all(np.abs(q) <= qmax)
    qg = np.abs(q).reshape(N, K // G, G).max(-1)
    wg = np.abs(W).reshape(N, K // G, G).max(-1)
    # the largest element of every non-zero group lands on +-qmax
    assert np.all(qg[wg > 0] == qmax)
    assert np.all(s[wg == 0] == 0) and np.all(qg[wg == 0] == 0)
    # error within half a step of the stored scale
    sk = np.repeat(s, G, axis=1)
    err = np.abs(q * sk - W.astype(np.float64))
    assert np.all(err <= 0.5 * sk)
    # the stored scale is amax/qmax rounded to bf16: within half a bf16 ulp (2^-8 relative)
    ratio = s[wg > 0] / (wg[wg > 0] / qmax)
    assert np.all(np.abs(ratio - 1) <= 2.0 ** -8)
    # dequant = q * s exactly
    dq = orc.dequant(fmt, codes, scales, None, N, K, G)
    assert np.array_equal(dq.astype(np.float64), q * sk)


@pytest.mark.parametrize("fmt,qmax", [("int2_sym", 1), ("int3_sym", 3), ("int4_sym", 7),
                                      ("int8_sym", 127)])
@pytest.mark.parametrize("sval", [1.0, 2.0 ** -7, 0.0173])
def test_sym_round_trip_every_code(orc, fmt, qmax, sval):
    """W = q*s for every representable q gives back q and s exactly."""
    s = float(oracle.bits_to_f32(np.array([orc.f64_to_bf16(sval)], np.uint16))[0])
    G = 256
    q = np.arange(-qmax, qmax + 1)
    row = np.resize(q, G).astype(np.float64)
    W = (row * s).astype(np.float32)[None, :].repeat(2, 0)
    codes, scales, _ = orc.quantize(fmt, W, G)
    assert np.all(_bf16(scales) == s)
    got = _signed_codes(fmt, codes)
    assert np.array_equal(got[0], row.astype(np.int64))


# --------------------------------------------------------------- asymmetric INT4
@pytest.mark.parametrize("G", [32, 128])
def test_asym_properties(orc, G):
    N, K = 48, 512
    W = _weights(N, K, seed=100 + G)
    W[2, :] = np.abs(W[2, :])      # groups with min > 0 (lo clamps to 0)
    W[3, :] = -np.abs(W[3, :])     # groups with max < 0
    codes, scales, zeros = orc.quantize("int4_asym", W, G)
    q = _nibbles(codes).astype(np.int64)
    s = _bf16(scales)
    z = zeros.astype(np.int64)
    assert q.min() >= 0 and q.max() <= 15 and z.min() >= 0 and z.max() <= 15
    w64 = W.astype(np.float64)
    lo = np.minimum(0, w64.reshape(N, K // G, G).min(-1))
    hi = np.maximum(0, w64.reshape(N, K // G, G).max(-1))
    s32 = (hi - lo) / 15.0
    # error bound: half a step, plus the bf16 rounding of the scale for clamped codes
    sk = np.repeat(s, G, axis=1)
    zk = np.repeat(z, G, axis=1)
    allow = 0.5 * sk + 15 * np.repeat(np.abs(s32 - s), G, axis=1) + 1e-12
    dq = orc.dequant("int4_asym", codes, scales, zeros, N, K, G)
    assert np.array_equal(dq.astype(np.float64), (q - zk) * sk)
    assert np.all(np.abs(dq - w64) <= allow)
    nz = hi - lo > 0
    assert np.all(np.abs(s[nz] / s32[nz] - 1) <= 2.0 ** -8)
    assert np.all(s[~nz] == 0)


def test_asym_round_trip(orc):
    """W = (q - z)*s with every q in 0..15 present gives back q, z and s."""
    G = 64
    rows = []
    for z in range(16):
        q = np.resize(np.arange(16), G)
        rows.append((q - z) * 0.03125)
    W = np.array(rows, dtype=np.float32)
    codes, scales, zeros = orc.quantize("int4_asym", W, G)
    assert np.all(_bf16(scales) == 0.03125)
    assert np.array_equal(zeros[:, 0], np.arange(16))
    assert np.array_equal(_nibbles(codes), np.resize(np.arange(16), (16, G)))


# --------------------------------------------------------------- Lloyd-Max
def _max_table():
    levels, mse = [], None
    with open(os.path.join(GOLDEN, "lloyd_max_gaussian16.txt")) as f:
        for line in f:
            if line.startswith("level"):
                levels.append(float(line.split()[1]))
            elif line.startswith("mse"):
                mse = float(line.split()[1])
    return np.array(levels), mse


def test_lloyd_max_invariants(orc):
    c64, c32, iters, mse = orc.lloyd_max(16)
    assert np.all(np.diff(c64) > 0)
    assert np.max(np.abs(c64 + c64[::-1])) < 1e-12          # symmetric
    assert np.array_equal(c32, c64.astype(np.float32))       # fp32 = RN(fp64)
    t = np.concatenate([[-np.inf], (c64[1:] + c64[:-1]) / 2, [np.inf]])
    q_mse = 0.0
    for i in range(16):
        mass = stats.norm.cdf(t[i + 1]) - stats.norm.cdf(t[i])
        mean, _ = integrate.quad(lambda x: x * stats.norm.pdf(x), t[i], t[i + 1],
                                 epsabs=1e-14, epsrel=1e-12)
        assert abs(mean / mass - c64[i]) < 1e-9               # centroid condition
        v, _ = integrate.quad(lambda x: (x - c64[i]) ** 2 * stats.norm.pdf(x), t[i], t[i + 1],
                              epsabs=1e-15, epsrel=1e-12)
        q_mse += v
    assert abs(q_mse - mse) < 1e-10
    levels, mse_tab = _max_table()
    assert np.max(np.abs(c64[8:] - levels)) < 1e-3
    assert abs(mse - mse_tab) < 1e-5


# --------------------------------------------------------------- codebook
def test_cb4_nearest_neighbour(orc):
    N, K = 40, 256
    W = _weights(N, K, seed=9)
    _, c32, _, _ = orc.lloyd_max(16)
    codes, norms, cent = orc.quantize("cb4", W, centroids=c32)
    idx = _nibbles(codes).astype(np.int64)
    nrm = _bf16(norms)
    ref_norm = np.linalg.norm(W.astype(np.float64), axis=1) / np.sqrt(K)
    nz = ref_norm > 0
    assert np.all(np.abs(nrm[nz] / ref_norm[nz] - 1) <= 2.0 ** -8)
    assert np.all(nrm[~nz] == 0) and np.all(idx[~nz] == 0)
    r = W[nz].astype(np.float64) / nrm[nz][:, None]
    d = np.abs(r[..., None] - c32.astype(np.float64)[None, None, :])
    best = d.argmin(-1)     # first minimum = lower index on ties
    assert np.array_equal(idx[nz], best)
    dq = orc.dequant("cb4", codes, norms, cent, N, K)
    want = (c32.astype(np.float64)[idx] * nrm[:, None]).astype(np.float32)
    assert np.array_equal(dq, want)


# --------------------------------------------------------------- NVFP4
def test_nvfp4_properties(orc):
    N, K = 64, 512
    W = (0.02 * synth.student5_stream(3, 1, 0, N * K)).astype(np.float32).reshape(N, K)
    W[5, 32:48] = 0.0              # an all-zero block
    codes, bs, ts = orc.quantize("nvfp4", W)
    q = _nibbles(codes).astype(np.int64)
    assert not np.any(q == 8)                       # no negative zero
    assert np.all(bs < 0x7F)                        # sign clear, never NaN
    amax = np.abs(W.astype(np.float64)).max()
    assert ts[0] == np.float32(amax / 2688.0)
    mag = np.array(E2M1)[q & 7]
    sgn = np.where(q & 8, -1.0, 1.0)
    sbv = np.array([orc.e4m3_value(int(c)) for c in range(128)])[bs.astype(np.int64)]
    sbk = np.repeat(sbv, 16, axis=1)
    dq_exact = sgn * mag * sbk * float(ts[0])
    dq = orc.dequant("nvfp4", codes, bs, ts, N, K)
    assert np.array_equal(dq, dq_exact.astype(np.float32))
    # the largest element of every block with a normal scale encodes to +-6
    blk_max = (q & 7).reshape(N, K // 16, 16).max(-1)
    normal = sbv >= 2.0 ** -6
    assert np.all(blk_max[normal] == 7)
    assert np.all(blk_max[sbv == 0] == 0)
    # error: at most half the E2M1 gap at the value's magnitude (gap 2 above 4)
    a = np.abs(W.astype(np.float64)) / (sbk * float(ts[0]) + (sbk == 0))
    gap = np.where(a <= 2, 0.5, np.where(a <= 4, 1.0, 2.0))
    err = np.abs(W.astype(np.float64) - dq_exact) / (sbk * float(ts[0]) + (sbk == 0))
    assert np.all(err[sbk > 0] <= 0.5 * gap[sbk > 0] + 1e-12)


# ------------------------------------------------------------------- MXFP4
def test_e8m0_values(orc):
    """E8M0: code c is 2^(c - 127); 255 is NaN (format definition)."""
    import math
    for c in range(255):
        assert orc.e8m0_value(c) == math.ldexp(1.0, c - 127)
    assert math.isnan(orc.e8m0_value(255))


def test_mxfp4_properties(orc):
    """Block scale = 2^(floor(log2 amax) - 2) from an independent frexp; every
    code within half the E2M1 gap, or saturated at 6 when |w| / scale > 6;
    exact dequant; no negative zero; all-zero blocks get code 0."""
    import math
    N, K = 48, 512
    W = (0.02 * synth.student5_stream(5, 1, 0, N * K)).astype(np.float32).reshape(N, K)
    W[3, 64:96] = 0.0                 # an all-zero block
    W[4, 7] = 3.0e5                   # a block scale far above the others
    codes, bs, aux = orc.quantize("mxfp4", W)
    assert aux is None and bs.shape == (N, K // 32)
    q = _nibbles(codes).astype(np.int64)
    assert not np.any(q == 8)
    W64 = W.astype(np.float64)
    amax = np.abs(W64).reshape(N, K // 32, 32).max(-1)
    want = np.zeros_like(bs, dtype=np.int64)
    for (n, b), a in np.ndenumerate(amax):
        if a > 0:
            want[n, b] = min(max(math.frexp(a)[1] - 1 - 2, -127), 127) + 127
    assert np.array_equal(bs.astype(np.int64), want)
    assert bs[3, 2] == 0 and not np.any(q[3, 64:96])
    X = np.repeat(np.ldexp(1.0, bs.astype(np.int64) - 127), 32, axis=1)
    mag = np.array(E2M1)[q & 7]
    dq_exact = np.where(q & 8, -1.0, 1.0) * mag * X
    dq = orc.dequant("mxfp4", codes, bs, None, N, K)
    assert np.array_equal(dq, dq_exact.astype(np.float32))
    a = np.abs(W64) / X
    gap = np.where(a <= 2, 0.5, np.where(a <= 4, 1.0, 2.0))
    err = np.abs(W64 - dq_exact) / X
    inside = a <= 6.0
    assert np.all(err[inside] <= 0.5 * gap[inside] + 1e-12)
    # above 6 the element saturates to +-6 (a block's largest is below 8)
    assert np.all(a < 8.0)
    assert np.all(np.abs(dq_exact[~inside]) == 6.0 * X[~inside])


def test_mxfp4_round_trip(orc):
    """Blocks built from E2M1 values times a power of two (each block holding
    +-6 at its scale) quantize back to the same codes and scale."""
    rng = np.random.default_rng(11)
    N, K = 8, 256
    e = rng.integers(100, 140, size=(N, K // 32))
    q = rng.integers(0, 16, size=(N, K))
    q[q == 8] = 0
    q[:, ::32] = 7                    # +6 in every block
    X = np.repeat(np.ldexp(1.0, e - 127), 32, axis=1)
    W = (np.where(q & 8, -1.0, 1.0) * np.array(E2M1)[q & 7] * X).astype(np.float32)
    codes, bs, _ = orc.quantize("mxfp4", W)
    assert np.array_equal(bs.astype(np.int64), e)
    assert np.array_equal(_nibbles(codes).astype(np.int64), q)


# ------------------------------------------------------------------ FP8 E4M3
FP8_MAX = {"fp8_e4m3": 448.0, "fp8_e5m2": 57344.0}


def _e4m3_table(fmt="fp8_e4m3"):
    """value of every code from torch's float8_e4m3fn / float8_e5m2 (an
    independent decoder)."""
    import torch
    dt = torch.float8_e4m3fn if fmt == "fp8_e4m3" else torch.float8_e5m2
    return torch.arange(256, dtype=torch.uint8).view(dt).to(torch.float64).numpy()


@pytest.mark.parametrize("G", [32, 128])
@pytest.mark.parametrize("fmt", ["fp8_e4m3", "fp8_e5m2"])
def test_fp8_properties(orc, G, fmt):
    """Group scale within half an fp32 ulp of amax/fmax (448 for E4M3, 57344
    for E5M2); every code the nearest finite value to w/s by brute force
    (ties to the even code), with the sign of w and +0 for zero; the group
    maximum at +-fmax; all-zero groups get scale 0 and code 0; dequant = fp32
    of the exact product."""
    from fractions import Fraction
    N, K = 24, 512
    W = _weights(N, K, seed=9)
    fmax = FP8_MAX[fmt]
    codes, scales, aux = orc.quantize(fmt, W, G)
    assert aux is None and codes.shape == (N, K) and scales.dtype == np.float32
    ng = K // G
    W64 = W.astype(np.float64)
    amax = np.abs(W64).reshape(N, ng, G).max(-1)
    for (n, j), a in np.ndenumerate(amax):
        s = scales[n, j]
        if a == 0.0:
            assert s == 0.0 and not np.any(codes[n, j * G:(j + 1) * G])
            continue
        exact = Fraction(a) / Fraction(fmax)
        ulp = np.spacing(np.float32(s))
        assert abs(Fraction(float(s)) - exact) <= Fraction(float(ulp)) / 2
    tab = _e4m3_table(fmt)
    fin = np.array([c for c in range(256) if np.isfinite(tab[c])])
    vals = tab[fin]
    S = np.repeat(scales.astype(np.float64), G, axis=1)
    live = S > 0
    r = np.where(live, W64 / np.where(live, S, 1.0), 0.0)
    # nearest finite value; among equals the code with an even mantissa
    d = np.abs(r[..., None] - vals[None, None, :])
    best = d.min(-1, keepdims=True)
    cand = d == best
    even = (fin & 1) == 0
    pick = np.where(cand & even[None, None, :], 1, 0) + cand
    want = fin[np.argmax(pick, axis=-1)]
    want = np.where(tab[want] == 0.0, 0, want)       # zero is written as +0
    got = codes.astype(np.int64)
    assert np.array_equal(got[live], want[live])
    gmax = np.abs(tab[got]).reshape(N, ng, G).max(-1)
    assert np.all(gmax[amax > 0] == fmax)
    dq = orc.dequant(fmt, codes, scales, None, N, K, G)
    assert np.array_equal(dq, (tab[got] * S).astype(np.float32))


def test_fp8_e4m3_round_trip(orc):
    """Groups built from E4M3 values (each holding +-448) times a power-of-two
    scale quantize back to the same codes and scale."""
    rng = np.random.default_rng(13)
    N, K, G = 8, 256, 64
    tab = _e4m3_table()
    fin = np.array([c for c in range(256) if np.isfinite(tab[c]) and c != 0x80])
    q = rng.choice(fin, size=(N, K))
    q[:, ::G] = 0x7E                   # +448 in every group
    s = np.ldexp(1.0, rng.integers(-20, -5, size=(N, K // G)))
    W = (tab[q] * np.repeat(s, G, axis=1)).astype(np.float32)
    codes, scales, _ = orc.quantize("fp8_e4m3", W, G)
    assert np.array_equal(scales.astype(np.float64), s)
    assert np.array_equal(codes.astype(np.int64), q)


def test_fp8_e5m2_round_trip(orc):
    """Groups built from E5M2 values (each holding +-57344) times a power-of-two
    scale quantize back to the same codes and scale."""
    rng = np.random.default_rng(14)
    N, K, G = 8, 256, 64
    tab = _e4m3_table("fp8_e5m2")
    fin = np.array([c for c in range(256) if np.isfinite(tab[c]) and c != 0x80])
    q = rng.choice(fin, size=(N, K))
    q[:, ::G] = 0x7B                   # +57344 in every group
    s = np.ldexp(1.0, rng.integers(-30, -16, size=(N, K // G)))
    W = (tab[q] * np.repeat(s, G, axis=1)).astype(np.float32)
    codes, scales, _ = orc.quantize("fp8_e5m2", W, G)
    assert np.array_equal(scales.astype(np.float64), s)
    assert np.array_equal(codes.astype(np.int64), q)
