"""GPU parity on small and ragged shapes: pack/unpack round trip, exact
dequant, the GPU quantizer against the oracle's, and the linear against the
oracle for every format, group size and a spread of batch sizes."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import (bf16_bits, check_close, dev_bf16, dev_u8, pack_on_gpu, run_linear,
                       small_case)

pytestmark = pytest.mark.gpu

FMT_G = [("int4_sym", 32), ("int4_sym", 64), ("int4_sym", 128), ("int4_sym", 256),
         ("int4_asym", 32), ("int4_asym", 128), ("int8_sym", 32), ("int8_sym", 256),
         ("cb4", 0), ("nvfp4", 16), ("mxfp4", 32), ("fp8_e4m3", 32), ("fp8_e4m3", 256),
         ("fp8_e5m2", 64), ("int2_sym", 32), ("int2_sym", 128), ("int3_sym", 32),
         ("int3_sym", 128)]
IDS = [f"{f}-g{g}" for f, g in FMT_G]


@pytest.mark.parametrize("fmt,G", FMT_G, ids=IDS)
def test_pack_unpack_round_trip(wq, orc, fmt, G):
    N, K = 48, 768 if G == 256 else 320
    K = K if (G == 0 or K % G == 0) else 768
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=3)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    cb, cs, ca = wq.wq_canonical_sizes(fmt, N, K, G)
    c2 = torch.zeros(cb, dtype=torch.uint8, device="cuda")
    s2 = torch.zeros(cs, dtype=torch.uint8, device="cuda")
    a2 = torch.zeros(max(ca, 16), dtype=torch.uint8, device="cuda") if ca else None
    wq.wq_unpack(fmt, N, K, G, pw.w, pw.scales, pw.aux, c2, s2, a2)
    torch.cuda.synchronize()
    assert np.array_equal(c2.cpu().numpy(), codes.view(np.uint8).reshape(-1))
    assert np.array_equal(s2.cpu().numpy(), scales.view(np.uint8).reshape(-1))
    if ca:
        assert np.array_equal(a2[:ca].cpu().numpy(), aux.view(np.uint8).reshape(-1))
    # the packed weight is a permutation: same multiset of bytes for 8-bit codes
    if fmt == "int8_sym":
        got = np.sort(pw.w.cpu().numpy() ^ 0x80)
        assert np.array_equal(got, np.sort(codes.view(np.uint8).reshape(-1)))


@pytest.mark.parametrize("fmt,G", FMT_G, ids=IDS)
def test_dequant_bit_exact(wq, orc, fmt, G):
    N, K = 64, 512
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=5)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    wq.wq_dequant(fmt, N, K, G, pw.w, pw.scales, pw.aux, out)
    torch.cuda.synchronize()
    ref = orc.dequant(fmt, codes, scales, aux, N, K, G)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("fmt,G", FMT_G, ids=IDS)
def test_gpu_quantizer_matches_oracle(wq, orc, fmt, G):
    N, K = 96, 1024
    W = synth.weight(17, N, K, dist="student5" if fmt in ("nvfp4", "mxfp4") else "normal", sigma=0.02,
                     outlier_count=100, outlier_mult=20.0)
    W[7, :] = 0.0
    W[9, 64:192] = 0.0
    codes, scales, aux = orc.quantize(fmt, W, G)
    cb, cs, ca = wq.wq_canonical_sizes(fmt, N, K, G)
    dc = torch.zeros(cb, dtype=torch.uint8, device="cuda")
    ds = torch.zeros(cs, dtype=torch.uint8, device="cuda")
    da = torch.zeros(max(ca, 16), dtype=torch.uint8, device="cuda") if ca else None
    if fmt == "cb4":
        da.view(torch.float32)[:16].copy_(torch.from_numpy(aux))
    wq.wq_quantize(fmt, N, K, G, torch.from_numpy(W).cuda(), dc, ds, da)
    torch.cuda.synchronize()
    assert np.array_equal(dc.cpu().numpy(), codes.view(np.uint8).reshape(-1))
    assert np.array_equal(ds.cpu().numpy(), scales.view(np.uint8).reshape(-1))
    if ca:
        assert np.array_equal(da[:ca].cpu().numpy(), aux.view(np.uint8).reshape(-1))


MS = [1, 2, 3, 4, 5, 7, 8, 9, 13, 16, 17, 31, 64, 100, 129, 300]


@pytest.mark.parametrize("fmt,G", FMT_G, ids=IDS)
@pytest.mark.parametrize("shape", [(80, 448), (256, 1024)], ids=["ragged80x448", "256x1024"])
def test_linear_parity(wq, orc, fmt, G, shape):
    N, K = shape
    if G and K % G:
        K = 1024
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=N + K)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    xa = synth.activations(31, max(MS), K)
    b = synth.bias(31, N)
    y_ref, _ = orc.linear(xa, dq, b)
    for M in MS:
        for bias in (b, None):
            y = run_linear(wq, pw, xa[:M], bias, M)
            ref = y_ref[:M] if bias is not None else orc.linear(xa[:M], dq, None)[0]
            check_close(y, ref, f"{fmt} g{G} N={N} K={K} M={M} bias={bias is not None}")


def _int_case(fmt, N, K, G, rng):
    import test_oracle_linear as tol
    return tol._int_case(fmt, N, K, G, rng)


@pytest.mark.parametrize("fmt,G", [("int4_sym", 64), ("int4_asym", 32), ("int8_sym", 128),
                                   ("cb4", 0), ("nvfp4", 16), ("mxfp4", 32), ("fp8_e4m3", 64),
                                   ("fp8_e5m2", 32), ("int2_sym", 64), ("int3_sym", 64)])
@pytest.mark.parametrize("M", [1, 5, 16, 40, 200])
def test_linear_integer_bit_exact(wq, orc, fmt, G, M):
    """Integer activations and unit scales: every partial sum is exact in
    fp32, so the GPU result must equal the oracle's bit for bit."""
    N, K = 96, 256
    rng = np.random.default_rng(7)
    codes, scales, aux, wval = _int_case(fmt, N, K, G, rng)
    if fmt == "cb4":   # keep |centroids| small enough that fp32 sums stay exact
        aux = ((np.arange(16) - 8) * 1.0).astype(np.float32)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    xi = rng.integers(-4, 5, size=(M, K))
    x = synth.f64_to_bf16_bits(xi.astype(np.float64))
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    ref, ref64 = orc.linear(x, dq, None)
    y = run_linear(wq, pw, x, None, M)
    assert np.array_equal(y, ref), f"max diff {np.max(np.abs(y.astype(int) - ref.astype(int)))}"


def test_linear_empty_and_api(wq, orc):
    N, K, G = 64, 256, 64
    W, (codes, scales, aux) = small_case(orc, "int4_sym", N, K, G, seed=1)
    pw = pack_on_gpu(wq, "int4_sym", N, K, G, codes, scales, aux)
    y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((1, K), dtype=torch.bfloat16, device="cuda")
    wq.wq_linear(x, pw.w, pw.scales, pw.aux, None, 0, N, K, "int4_sym", G, y)
    # the high-level helper, from host memory, matches the C call
    xa = synth.activations(2, 3, K)
    xh = torch.from_numpy(xa.view(np.int16).copy()).view(torch.bfloat16)
    yh = wq.linear(xh, pw)
    yd = run_linear(wq, pw, xa, None, 3)
    assert np.array_equal(bf16_bits(yh), yd)
    # quantize_and_pack on the GPU gives the same packed bytes as the oracle path
    pw2 = wq.quantize_and_pack(torch.from_numpy(W).cuda(), "int4_sym", G)
    assert torch.equal(pw2.w, pw.w) and torch.equal(pw2.scales, pw.scales)


def test_linear_respects_stream(wq, orc):
    N, K, G = 128, 512, 128
    W, (codes, scales, aux) = small_case(orc, "int4_asym", N, K, G, seed=2)
    pw = pack_on_gpu(wq, "int4_asym", N, K, G, codes, scales, aux)
    xa = synth.activations(3, 4, K)
    ref = run_linear(wq, pw, xa, None, 4)
    s = torch.cuda.Stream()
    x = dev_bf16(xa)
    y = torch.empty((4, N), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        wq.wq_linear(x, pw.w, pw.scales, pw.aux, None, 4, N, K, "int4_asym", G, y, s)
    s.synchronize()
    assert np.array_equal(bf16_bits(y), ref)


EDGE = [
    # (N, K, G, Ms): the smallest packed weight (one row tile, one 64-K block);
    # an odd number of scale groups; a long K whose activation slice forces a
    # six-block cluster at M = 16
    (16, 64, 32, (1, 7, 16, 17, 40)),
    (48, 192, 64, (3, 16, 33, 130)),
    (32, 16384, 256, (1, 16, 20)),
    # enough row groups for the eight-warp decode CTAs, with fewer K blocks
    # (three 4-bit blocks) than warps
    (19008, 192, 64, (1, 9, 16)),
]


@pytest.mark.parametrize("fmt", ["int4_sym", "int4_asym", "int8_sym", "cb4", "nvfp4", "mxfp4",
                                 "fp8_e4m3", "fp8_e5m2", "int2_sym", "int3_sym"])
@pytest.mark.parametrize("case", EDGE, ids=["16x64", "48x192", "32x16384", "19008x192"])
def test_linear_edge_shapes(wq, orc, fmt, case):
    N, K, G, Ms = case
    G = {"cb4": 0, "nvfp4": 16, "mxfp4": 32}.get(fmt, G)
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=N * 7 + K)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    xa = synth.activations(41, max(Ms), K)
    b = synth.bias(41, N)
    for M in Ms:
        y = run_linear(wq, pw, xa[:M], b, M)
        ref, _ = orc.linear(xa[:M], dq, b)
        check_close(y, ref, f"{fmt} N={N} K={K} M={M}")


@pytest.mark.parametrize("M", [8, 40])
def test_mxfp4_every_scale_code(wq, orc, M):
    """Every E8M0 code 0..254 and every E2M1 code, read through the linear with
    one-hot activations (y[m, n] is one weight, exactly): the smallest scales
    give bf16 subnormal weights, the largest overflow to inf, and code 255
    (NaN) or an inf weight times a zero activation makes the whole output
    column NaN, as in the fp64 definition."""
    N, K = 256, 512
    nb = K // 32
    rng = np.random.default_rng(11)
    q = rng.integers(0, 16, size=(N, K))
    import test_oracle_linear as tol
    codes = tol._pack_nibbles(q)
    e = (np.arange(N * nb).reshape(N, nb) % 255).astype(np.uint8)
    e[3, 5] = 255
    pw = pack_on_gpu(wq, "mxfp4", N, K, 32, codes, e, None)
    dq = orc.dequant("mxfp4", codes, e, None, N, K, 32)
    ks = (np.arange(M) * 37 + 5) % K
    xf = np.zeros((M, K))
    xf[np.arange(M), ks] = 1.0
    x = synth.f64_to_bf16_bits(xf)
    ref, _ = orc.linear(x, dq, None)
    y = run_linear(wq, pw, x, None, M)
    yf = oracle.bits_to_f32(y)
    rf = oracle.bits_to_f32(ref)
    assert np.array_equal(np.isnan(yf), np.isnan(rf))
    ok = ~np.isnan(rf)
    assert ok.sum() > 0.7 * ok.size
    assert np.array_equal(yf[ok], rf[ok])
    # the finite columns hold the weight itself, subnormals included
    w_sel = dq[:, ks].T
    assert np.array_equal(rf[ok], w_sel.astype(np.float32)[ok])
    assert (np.abs(w_sel[ok]) < 2.0 ** -126).any() and (np.abs(w_sel[ok]) > 2.0 ** 60).any()


@pytest.mark.parametrize("M", [8, 40])
@pytest.mark.parametrize("fmt", ["fp8_e4m3", "fp8_e5m2"])
def test_fp8_every_code(wq, orc, fmt, M):
    """Every finite FP8 code (subnormals, +-0 and the largest value included)
    read through the linear with one-hot activations: y[m, n] is one weight,
    exactly (bf16 holds every E4M3 and E5M2 value)."""
    N, K, G = 256, 512, 64
    rng = np.random.default_rng(12)
    if fmt == "fp8_e4m3":
        bad = (0x7F, 0xFF)
    else:
        bad = tuple(c for c in range(256) if (c >> 2) & 31 == 31)
    fin = np.array([c for c in range(256) if c not in bad], np.uint8)
    codes = fin[(np.arange(N * K) * 7 + rng.integers(0, 254)) % fin.size].reshape(N, K)
    scales = np.ldexp(1.0, rng.integers(-3, 4, size=(N, K // G))).astype(np.float32)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, None)
    dq = orc.dequant(fmt, codes, scales, None, N, K, G)
    ks = (np.arange(M) * 41 + 3) % K
    xf = np.zeros((M, K))
    xf[np.arange(M), ks] = 1.0
    x = synth.f64_to_bf16_bits(xf)
    ref, _ = orc.linear(x, dq, None)
    y = run_linear(wq, pw, x, None, M)
    assert np.array_equal(oracle.bits_to_f32(y), oracle.bits_to_f32(ref))
    assert np.array_equal(oracle.bits_to_f32(ref), dq[:, ks].T.astype(np.float32))


@pytest.mark.parametrize("fmt,G", [("int4_sym", 128), ("nvfp4", 16)])
def test_long_k_small_batch_takes_prefill(wq, orc, fmt, G):
    """K = 65536 at M = 16 does not fit the decode kernel's staged activation
    slice; the call runs the prefill kernel instead (M = 1 still decodes)."""
    N, K = 16, 65536
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=19)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    xa = synth.activations(61, 16, K)
    for M in (1, 16):
        y = run_linear(wq, pw, xa[:M], None, M)
        ref, _ = orc.linear(xa[:M], dq, None)
        check_close(y, ref, f"{fmt} long K M={M}")
