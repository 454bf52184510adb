"""GPU parity of the linear with a SwiGLU input ([up | gate] rows, activation
up * silu(gate) rounded to bf16): decode batches apply the step to the staged
activation slice, larger ones materialize it in the caller's workspace."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_cases import bf16_bits, check_close, dev_bf16, pack_on_gpu, small_case

pytestmark = pytest.mark.gpu

MS = [1, 3, 8, 16, 17, 64, 200]


def _run(wq, pw, x2_bits, bias_bits, M, ws_rows=None):
    x2 = dev_bf16(x2_bits)
    b = dev_bf16(bias_bits) if bias_bits is not None else None
    y = torch.full((max(M, 1), pw.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = None
    if M > 16 or ws_rows:
        ws = torch.full((ws_rows or M, pw.K), float("nan"), dtype=torch.bfloat16, device="cuda")
    wq.wq_linear_swiglu(x2, pw.w, pw.scales, pw.aux, b, M, pw.N, pw.K, pw.fmt, pw.group_size,
                        ws, 0 if ws is None else ws.numel() * 2, y)
    torch.cuda.synchronize()
    return bf16_bits(y[:M])


@pytest.mark.parametrize("fmt,G", [("int4_asym", 128), ("int8_sym", 64), ("nvfp4", 16),
                                   ("cb4", 0), ("fp8_e4m3", 32)])
def test_swiglu_linear_matches_oracle(wq, orc, fmt, G):
    N, K = 96, 1024
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=8)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    x2 = synth.activations(51, max(MS), 2 * K)
    b = synth.bias(51, N)
    a = orc.swiglu(x2)
    for M in MS:
        y = _run(wq, pw, x2[:M], b, M)
        ref, _ = orc.linear(a[:M], dq, b)
        check_close(y, ref, f"{fmt} swiglu M={M}")


def test_swiglu_equals_linear_on_materialized_activation(wq, orc):
    """The fused decode step and the materialized prefill step agree with
    wq_linear run on the oracle's bf16 activation (up to the rare bf16
    neighbours where fp32 and fp64 silu round differently)."""
    fmt, G, N, K = "int4_sym", 64, 64, 512
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=9)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    x2 = synth.activations(52, 40, 2 * K)
    a = orc.swiglu(x2)
    for M in (4, 40):
        y_sw = _run(wq, pw, x2[:M], None, M)
        y_lin = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        wq.wq_linear(dev_bf16(a[:M]), pw.w, pw.scales, pw.aux, None, M, N, K, fmt, G, y_lin)
        torch.cuda.synchronize()
        y_lin = bf16_bits(y_lin)
        check_close(y_sw, y_lin, f"swiglu vs linear M={M}")


def test_swiglu_helper_and_empty(wq, orc):
    fmt, G, N, K = "nvfp4", 16, 48, 256
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=10)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    x2 = synth.activations(53, 33, 2 * K)
    xt = dev_bf16(x2).reshape(3, 11, 2 * K)
    y = wq.linear_swiglu(xt, pw)
    assert y.shape == (3, 11, N)
    ref, _ = orc.linear(orc.swiglu(x2), orc.dequant(fmt, codes, scales, aux, N, K, G), None)
    check_close(bf16_bits(y.reshape(33, N)), ref, "linear_swiglu helper")
    # M = 0: nothing launched, output untouched
    out = torch.full((1, N), 7.0, dtype=torch.bfloat16, device="cuda")
    wq.wq_linear_swiglu(dev_bf16(x2[:1]), pw.w, pw.scales, pw.aux, None, 0, N, K, fmt, G, None,
                        0, out)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_swiglu_long_k_small_batch(wq, orc):
    """M <= 16 with a K too long to stage both halves: with a workspace the
    activation is materialized and the prefill kernel runs; without one the
    call is refused (nothing launched)."""
    fmt, G, N, K = "int4_asym", 128, 16, 65536
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=20)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    M = 16
    x2 = synth.activations(62, M, 2 * K)
    ref, _ = orc.linear(orc.swiglu(x2), dq, None)
    y = _run(wq, pw, x2, None, M, ws_rows=M)
    check_close(y, ref, "swiglu long K")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wq.WQError) as ei:
        wq.wq_linear_swiglu(dev_bf16(x2), pw.w, pw.scales, pw.aux, None, M, N, K, fmt, G, None, 0,
                            out)
    assert ei.value.status == wq.WQ_ERR_UNSUPPORTED
