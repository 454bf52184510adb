"""GPU parity of the activation-quantized linear (per-token INT8 activations,
INT8 weight codes, tcgen05.mma.kind::i8 with exact s32 group sums): the
activation codes and scales equal the oracle's bit for bit, and every output
is within the parity tolerance of the oracle's activation-quantized linear
(its own reference, not the weight-only one), with output canaries."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
import synth.workloads as W
from gpu_cases import (bf16_bits, check_close, check_guards, dev_bf16, dev_u8, guarded_out,
                       pack_on_gpu, small_case)

pytestmark = pytest.mark.gpu


def _run_a8(wq, pw, x_bits, bias_bits, M):
    x = dev_bf16(x_bits)
    b = dev_bf16(bias_bits) if bias_bits is not None else None
    need = wq.wq_linear_a8_workspace_size(M, pw.K)
    ws = torch.full((max(need, 16),), 0x5A, dtype=torch.uint8, device="cuda")
    buf, y = guarded_out(M, pw.N)
    wq.wq_linear_a8(x, pw.w, pw.scales, b, M, pw.N, pw.K, pw.fmt, pw.group_size, ws, need, y)
    torch.cuda.synchronize()
    check_guards(buf, M, pw.N, f"a8 M={M} N={pw.N} K={pw.K}")
    assert wq.wq_device_error() == 0
    return bf16_bits(y[:M])


@pytest.mark.parametrize("M,K", [(1, 1024), (5, 512), (64, 4096), (300, 2048), (33, 8192)])
def test_activation_codes_bit_exact(wq, orc, M, K):
    x = synth.activations(70 + M, M, K, channel_count=max(1, K // 100), channel_mult=10.0)
    if M > 2:
        x[1] = 0                                         # an all-zero token: scale 0, codes 0
    xq_ref, sx_ref = orc.quant_act_int8(x)
    xq = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    sx = torch.zeros((M,), dtype=torch.float32, device="cuda")
    wq.wq_quantize_act_int8(dev_bf16(x), M, K, xq, sx)
    torch.cuda.synchronize()
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), sx_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)


@pytest.mark.parametrize("fmt", ["int8_sym", "int4_sym"])
@pytest.mark.parametrize("G", [32, 64, 128, 256])
@pytest.mark.parametrize("M", [1, 16, 40, 128, 200, 300])
def test_a8_linear_matches_oracle(wq, orc, fmt, G, M):
    """W8A8 and W4A8 (INT4 codes used as INT8) against the oracle."""
    N, K = 272, 1024
    Wd, (codes, scales, _) = small_case(orc, fmt, N, K, G, seed=71)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, None)
    x = synth.activations(72, M, K, channel_count=10, channel_mult=10.0)
    b = synth.bias(71, N) if M % 2 == 0 else None
    y = _run_a8(wq, pw, x, b, M)
    ref, _ = orc.linear_a8(fmt, codes, scales, N, K, G, x, b)
    check_close(y, ref, f"a8 {fmt} G={G} M={M}")


def test_a8_split_k_cluster(wq, orc):
    """Few output tiles and a long K: the K range is split over a cluster and
    the partial tiles summed through distributed shared memory."""
    N, K, G, M = 128, 8192, 256, 256
    Wd, (codes, scales, _) = small_case(orc, "int8_sym", N, K, G, seed=73)
    pw = pack_on_gpu(wq, "int8_sym", N, K, G, codes, scales, None)
    x = synth.activations(74, M, K)
    b = synth.bias(73, N)
    y = _run_a8(wq, pw, x, b, M)
    ref, _ = orc.linear_a8_full(codes, scales, N, K, G, x, b)
    check_close(y, ref, "a8 split-K")


@pytest.mark.parametrize("fmt", ["int8_sym", "int4_sym"])
def test_a8_integer_case_bit_exact(wq, orc, fmt):
    """Unit weight scales, activations on the INT8 grid with row maximum 127
    (s_x = 1): every output is an exact integer below 2^24, so the GPU result
    equals the oracle's bit for bit (every INT4 code, -8 included)."""
    N, K, G, M = 256, 512, 128, 70
    rng = np.random.default_rng(75)
    scales = np.full((N, K // G), 0x3F80, np.uint16)
    if fmt == "int8_sym":
        q = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    else:
        v = rng.integers(-8, 8, size=(N, K))
        q = ((v[:, 0::2] & 15) | ((v[:, 1::2] & 15) << 4)).astype(np.uint8)
    pw = pack_on_gpu(wq, fmt, N, K, G, q, scales, None)
    xi = rng.integers(-3, 4, size=(M, K))
    xi[:, 5] = 127
    x = synth.f64_to_bf16_bits(xi.astype(np.float64))
    y = _run_a8(wq, pw, x, None, M)
    ref, _ = orc.linear_a8_full(q, scales, N, K, G, x, None)
    assert np.array_equal(y, ref)


def test_a8_full_size_prefill_layer(wq, orc):
    """The INT8 g256 8192 x 8192 layer at M = 1024, 2048, 4096, every output
    against the oracle's activation-quantized linear."""
    wl = W.PREFILL
    Wd = W.make_weight(wl)
    codes, scales, _ = orc.quantize(wl.fmt, Wd, wl.group_size)
    pw = pack_on_gpu(wq, wl.fmt, wl.N, wl.K, wl.group_size, codes, scales, None)
    xa = W.make_x(wl, max(wl.Ms))
    b = W.make_bias(wl)
    for M in wl.Ms:
        y = _run_a8(wq, pw, xa[:M], b, M)
        ref, _ = orc.linear_a8_full(codes, scales, wl.N, wl.K, wl.group_size, xa[:M], b)
        check_close(y, ref, f"a8 full size M={M}")


def test_a8_refuses_other_formats(wq, orc):
    N, K, G, M = 64, 512, 64, 20
    Wd, (codes, scales, _) = small_case(orc, "int2_sym", N, K, G, seed=76)
    pw = pack_on_gpu(wq, "int2_sym", N, K, G, codes, scales, None)
    x = dev_bf16(synth.activations(77, M, K))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    need = wq.wq_linear_a8_workspace_size(M, K)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    with pytest.raises(wq.WQError) as ei:
        wq.wq_linear_a8(x, pw.w, pw.scales, None, M, N, K, "int2_sym", G, ws, need, y)
    assert ei.value.status == wq.WQ_ERR_UNSUPPORTED


def test_public_linear_a8(wq, orc):
    N, K, G = 128, 1024, 128
    Wd, (codes, scales, _) = small_case(orc, "int8_sym", N, K, G, seed=78)
    pw = pack_on_gpu(wq, "int8_sym", N, K, G, codes, scales, None)
    x = synth.activations(79, 2 * 3 * 7, K).reshape(2, 21, K)
    y = wq.linear_a8(dev_bf16(x), pw)
    assert y.shape == (2, 21, N)
    ref, _ = orc.linear_a8("int8_sym", codes, scales, N, K, G, x.reshape(-1, K))
    check_close(bf16_bits(y.reshape(-1, N)), ref, "public linear_a8")
