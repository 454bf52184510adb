"""wq_linear_swiglu_static: the SwiGLU-input linear with its activation
materialized in the library's static device scratch instead of a caller
workspace.  CPU: the symbol is exported and oversized or bad requests are
refused before anything launches.  GPU: results identical to
wq_linear_swiglu with a caller workspace, and no device memory allocated."""
from __future__ import annotations

import gc

import numpy as np
import pytest

import mixed_gemm_b200 as wqm

SCRATCH = 16 << 20


def test_static_entry_exported_and_refuses_oversize():
    base = 1 << 20
    f = wqm.FORMATS["int4_sym"]
    N, K, G = 256, 8192, 64
    M = SCRATCH // (2 * K) + 1          # one row more than the scratch holds
    assert wqm._lib.wq_linear_swiglu_static(base, base * 64, base * 128, None, None, M, N, K, f,
                                            G, base * 4096, 0) == wqm.WQ_ERR_UNSUPPORTED
    # argument checks as wq_linear_swiglu (misaligned output, bad group)
    assert wqm._lib.wq_linear_swiglu_static(base, base * 64, base * 128, None, None, 32, N, K, f,
                                            G, base * 4096 + 8, 0) == wqm.WQ_ERR_ALIGNMENT
    assert wqm._lib.wq_linear_swiglu_static(base, base * 64, base * 128, None, None, 32, N, K, f,
                                            48, base * 4096, 0) == wqm.WQ_ERR_INVALID_ARG


@pytest.mark.gpu
def test_static_scratch_matches_workspace_and_allocates_nothing(orc):
    import torch

    import synth
    from gpu_cases import bf16_bits, dev_bf16, pack_on_gpu, small_case

    fmt, G, N, K = "int4_asym", 128, 128, 1024
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=15)
    pw = pack_on_gpu(wqm, fmt, N, K, G, codes, scales, aux)
    x2 = dev_bf16(synth.activations(54, 300, 2 * K))
    for M in (8, 64, 300):
        y_ws = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty((max(M, 17), K), dtype=torch.bfloat16, device="cuda")
        wqm.wq_linear_swiglu(x2[:M], pw.w, pw.scales, pw.aux, None, M, N, K, fmt, G, ws,
                             ws.numel() * 2, y_ws)
        y_st = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        wqm.wq_linear_swiglu_static(x2[:M], pw.w, pw.scales, pw.aux, None, M, N, K, fmt, G,
                                    y_st)                      # warm-up: module and scratch loaded
        torch.cuda.synchronize()
        gc.collect()                 # tensors of earlier tests may be freed meanwhile
        free0, _ = torch.cuda.mem_get_info()
        alloc0 = torch.cuda.memory_allocated()
        for _ in range(3):
            wqm.wq_linear_swiglu_static(x2[:M], pw.w, pw.scales, pw.aux, None, M, N, K, fmt, G,
                                        y_st)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        # no device memory taken by the calls (torch's own count may only fall)
        assert free1 == free0 and torch.cuda.memory_allocated() <= alloc0
        assert np.array_equal(bf16_bits(y_st), bf16_bits(y_ws)), f"M={M}"


@pytest.mark.gpu
def test_static_scratch_on_the_decode_fallback(orc):
    """A batch of at most 16 rows whose K is too long for the decode kernel's
    staged slice (here 16 x 65536 with both SwiGLU halves) takes the
    materialized path, so the static scratch is used there too: identical to
    the caller-workspace call on two calls in a row, within the parity
    tolerance of the oracle, and no device memory allocated."""
    import torch

    import synth
    from gpu_cases import bf16_bits, check_close, dev_bf16, pack_on_gpu, small_case

    fmt, G, N, K, M = "int4_sym", 128, 128, 65536, 16
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=16)
    pw = pack_on_gpu(wqm, fmt, N, K, G, codes, scales, aux)
    x2h = synth.activations(55, M, 2 * K)
    x2 = dev_bf16(x2h)
    # the decode kernel refuses this shape: without a workspace the call is unsupported
    y_none = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = wqm._lib.wq_linear_swiglu(x2.data_ptr(), pw.w.data_ptr(), pw.scales.data_ptr(), None,
                                   None, M, N, K, wqm.FORMATS[fmt], G, None, 0,
                                   y_none.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == wqm.WQ_ERR_UNSUPPORTED
    y_ws = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    wqm.wq_linear_swiglu(x2, pw.w, pw.scales, pw.aux, None, M, N, K, fmt, G, ws, ws.numel() * 2,
                         y_ws)
    y_st = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    wqm.wq_linear_swiglu_static(x2, pw.w, pw.scales, pw.aux, None, M, N, K, fmt, G, y_st)
    torch.cuda.synchronize()
    gc.collect()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(2):
        y_st.fill_(float("nan"))
        wqm.wq_linear_swiglu_static(x2, pw.w, pw.scales, pw.aux, None, M, N, K, fmt, G, y_st)
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(y_st), bf16_bits(y_ws))
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0 and torch.cuda.memory_allocated() <= alloc0
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    ref, _ = orc.linear(orc.swiglu(x2h), dq, None)
    check_close(bf16_bits(y_st), ref, "static scratch, decode fallback")
