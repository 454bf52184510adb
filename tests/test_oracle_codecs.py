"""Pins of the oracle's scalar codecs (bf16, E2M1, E4M3) against things other
than the oracle itself: the format tables, torch's own casts, exact rational
rounding."""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_pairs(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            rows.append((a, b))
    return rows


# ------------------------------------------------------------------ bf16
def test_bf16_from_f32_matches_torch(orc):
    """Every fp32 input (incl. exact ties, subnormals, overflow) rounds as torch rounds."""
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    ties = (bits & np.uint32(0xFFFF0000)) | np.uint32(0x8000)   # exactly half-way
    specials = np.array([0x00000000, 0x80000000, 0x00000001, 0x007FFFFF, 0x00800000,
                         0x7F7FFFFF, 0x7F7F8000, 0x7F7F7FFF, 0x3F808000, 0x3F818000,
                         0x3F800001, 0xBF808000], dtype=np.uint32)
    allb = np.concatenate([bits, ties, specials])
    f = allb.view(np.float32)
    f = f[np.isfinite(f)]
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.f64_to_bf16(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(got, ref)


def _bf16_exact_rne(v: Fraction) -> Fraction:
    """Correct bf16 rounding of an exact rational (8 significant bits, ties even)."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix e so that 2^e <= a < 2^(e+1)
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


def test_bf16_from_f64_is_correctly_rounded(orc):
    """Doubles that are not fp32 values: the single rounding is the exact one."""
    import synth
    rng = np.random.default_rng(11)
    vals = rng.standard_normal(3000) * np.exp2(rng.integers(-140, 120, size=3000))
    # doubles just off a bf16 half-way point, where a double rounding would go wrong
    mids = (1.0 + np.arange(1, 200) / 128.0 + 1.0 / 256.0) * (1 + 2.0 ** -40)
    vals = np.concatenate([vals, mids, -mids])
    got = np.array([orc.f64_to_bf16(float(v)) for v in vals], dtype=np.uint16)
    for v, g in zip(vals, got):
        want = _bf16_exact_rne(Fraction(float(v)))
        gv = Fraction(float(orc.bf16_to_f32(int(g))))
        assert gv == want, (v, g)
    # the input generator's own rounding (a separate implementation) agrees
    assert np.array_equal(synth.f64_to_bf16_bits(vals), got)


# ------------------------------------------------------------------ E2M1
def test_e2m1_value_table(orc):
    for code, val in _read_pairs("e2m1_table.txt"):
        got = orc.e2m1_value(int(code))
        assert got == float(val)
        assert math.copysign(1.0, got) == math.copysign(1.0, float(val))


def test_e2m1_ties_and_saturation(orc):
    for val, code in _read_pairs("e2m1_rne_ties.txt"):
        assert orc.e2m1_encode(float(val)) == int(code), val


def test_e2m1_round_trip_every_code(orc):
    for code in range(16):
        back = orc.e2m1_encode(orc.e2m1_value(code))
        assert back == (0 if code == 8 else code)   # -0 is written as +0


def test_e2m1_encode_is_nearest(orc):
    """Brute force: the chosen code is a nearest table entry for random inputs."""
    vals = [orc.e2m1_value(c) for c in range(16)]
    rng = np.random.default_rng(3)
    for r in rng.uniform(-8, 8, size=4000):
        c = orc.e2m1_encode(float(r))
        d = abs(vals[c] - r)
        assert all(d <= abs(v - r) + 0.0 for v in vals), (r, c)
        if abs(r) < 0.25:
            assert c == 0


# ------------------------------------------------------------------ E4M3
def test_e4m3_values_match_torch(orc):
    codes = np.arange(0, 127, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.e4m3_value(int(c)) for c in codes])
    assert np.array_equal(got, ref)
    assert orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x01) == 2.0 ** -9
    assert math.isnan(orc.e4m3_value(0x7F))
    assert np.all(np.diff(got) > 0)   # monotone in the code


def test_e4m3_encode_matches_torch_in_range(orc):
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.uniform(0, 448, 3000), np.exp2(rng.uniform(-12, 8.8, 3000))])
    v = v[v <= 448].astype(np.float32).astype(np.float64)   # fp32 inputs: torch casts from fp32
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(float(x)) for x in v], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_round_trip_and_saturation(orc):
    for c in range(127):
        assert orc.e4m3_encode(orc.e4m3_value(c)) == c
    assert orc.e4m3_encode(448.0) == 0x7E
    assert orc.e4m3_encode(1e9) == 0x7E
    assert orc.e4m3_encode(0.0) == 0
    assert orc.e4m3_encode(2.0 ** -10) == 0      # tie between 0 and 2^-9: even code 0
    assert orc.e4m3_encode(3 * 2.0 ** -10) == 2  # tie between codes 1 and 2: even


@pytest.mark.parametrize("code", [0x00, 0x38, 0x7E])
def test_e4m3_named_points(orc, code):
    assert orc.e4m3_value(code) == {0x00: 0.0, 0x38: 1.0, 0x7E: 448.0}[code]


def test_e5m2_values_match_torch(orc):
    codes = np.arange(0, 256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e5m2).to(torch.float64).numpy()
    got = np.array([orc.e5m2_value(int(c)) for c in codes])
    fin = np.isfinite(ref)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(ref)], ref[~np.isnan(ref)])   # +-inf included
    assert orc.e5m2_value(0x7B) == 57344.0
    assert orc.e5m2_value(0x01) == 2.0 ** -16
    assert np.all(np.diff(got[:0x7C]) > 0)
    assert fin.sum() == 248


def test_e5m2_encode_matches_torch_in_range(orc):
    rng = np.random.default_rng(6)
    v = np.concatenate([rng.uniform(0, 57344, 3000), np.exp2(rng.uniform(-18, 15.8, 3000))])
    v = v[v <= 57344].astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e5m2).view(torch.uint8).numpy()
    got = np.array([orc.e5m2_encode(float(x)) for x in v], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e5m2_round_trip_and_saturation(orc):
    for c in range(0x7C):
        assert orc.e5m2_encode(orc.e5m2_value(c)) == c
    assert orc.e5m2_encode(57344.0) == 0x7B
    assert orc.e5m2_encode(1e30) == 0x7B
    assert orc.e5m2_encode(0.0) == 0
    assert orc.e5m2_encode(2.0 ** -17) == 0       # tie between 0 and 2^-16: even code 0
    assert orc.e5m2_encode(3 * 2.0 ** -17) == 2   # tie between codes 1 and 2: even
