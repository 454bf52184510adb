"""Stream-order guarantees of the library on the GPU.

The decode kernel is launched with programmatic dependent launch and requests
its packed weights before it waits for the previous kernel on the stream, so
every library call that writes packed weights ends with a stream operation
that is not a kernel.  These tests enqueue a weight writer and a linear that
reads its result back to back on one stream, with no host synchronization in
between, and compare with the oracle.  They also run the public ``linear`` on
a side stream with host activations, and first calls of new kernel
instantiations from several host threads at once (kernel attributes are set
per device under a lock)."""
from __future__ import annotations

import threading

import numpy as np
import pytest
import torch

import synth
from gpu_cases import bf16_bits, check_close, dev_bf16, dev_u8, small_case

pytestmark = pytest.mark.gpu


def test_pack_then_decode_on_one_stream(wq, orc):
    fmt, G, N, K, M = "int4_asym", 128, 512, 4096, 4
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=61)
    cw, cs, ca = dev_u8(codes), dev_u8(scales), dev_u8(aux)
    x = synth.activations(61, M, K)
    xd = dev_bf16(x)
    s = torch.cuda.Stream()
    wb, sb, ab = wq.wq_packed_sizes(fmt, N, K, G)
    torch.cuda.synchronize()
    for rep in range(3):
        pw_, ps_, pa_ = (torch.zeros(max(n, 16), dtype=torch.uint8, device="cuda")
                         for n in (wb, sb, ab))
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        # a long kernel first, so the pack would still be running if the linear
        # started early
        with torch.cuda.stream(s):
            torch.cuda._sleep(2_000_000)
        wq.wq_pack(fmt, N, K, G, cw, cs, ca, pw_, ps_, pa_, s)
        wq.wq_linear(xd, pw_, ps_, pa_, None, M, N, K, fmt, G, y, s)
        s.synchronize()
        dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
        ref, _ = orc.linear(x, dq, None)
        check_close(bf16_bits(y), ref, f"pack -> linear, rep {rep}")


@pytest.mark.parametrize("seed", [None, 77])
def test_lora_merge_then_decode_on_one_stream(wq, orc, seed):
    fmt, G, N, K, R, M = "int8_sym", 128, 256, 2048, 8, 8
    W, (codes, scales, _) = small_case(orc, fmt, N, K, G, seed=62)
    pw = wq.pack(fmt, N, K, G, dev_u8(codes), dev_u8(scales), None)
    m1 = synth.activations(63, N, R, sigma=0.3)
    m2 = synth.activations(64, R, K, sigma=0.3)
    x = synth.activations(65, M, K)
    xd, d1, d2 = dev_bf16(x), dev_bf16(m1), dev_bf16(m2)
    y0 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    # linear on the old codes, merge in place, linear on the new codes: one
    # stream, no host synchronization
    wq.wq_linear(xd, pw.w, pw.scales, None, None, M, N, K, fmt, G, y0, s)
    wq.wq_addmm_requant(fmt, N, K, G, pw.w, pw.scales, d1, d2, R, 0.5, 1.0, seed, s)
    wq.wq_linear(xd, pw.w, pw.scales, None, None, M, N, K, fmt, G, y, s)
    s.synchronize()
    new_codes = orc.addmm_requant_int8(codes, scales, G, m1, m2, 0.5, 1.0, seed)
    assert not np.array_equal(new_codes, codes)
    ref_old, _ = orc.linear(x, orc.dequant(fmt, codes, scales, None, N, K, G), None)
    ref_new, _ = orc.linear(x, orc.dequant(fmt, new_codes, scales, None, N, K, G), None)
    check_close(bf16_bits(y0), ref_old, "before the merge")
    check_close(bf16_bits(y), ref_new, "after the merge")
    assert not np.array_equal(ref_old, ref_new)


def test_public_linear_host_input_on_side_stream(wq, orc):
    fmt, G, N, K = "nvfp4", 16, 384, 2048
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=66)
    pw = wq.pack(fmt, N, K, G, dev_u8(codes), dev_u8(scales), dev_u8(aux))
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    s = torch.cuda.Stream()
    for M in (3, 40):
        x = synth.activations(67 + M, M, K)
        xh = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
        with torch.cuda.stream(s):
            torch.cuda._sleep(1_000_000)   # the side stream is busy when the call is made
        y = wq.linear(xh, pw, stream=s)
        assert not y.is_cuda
        ref, _ = orc.linear(x, dq, None)
        check_close(y.view(torch.int16).numpy().view(np.uint16), ref, f"host x, side stream, M={M}")


def test_first_calls_from_several_threads(wq, orc):
    """Kernel instantiations used for the first time in this process, called
    from four host threads at once (each on its own stream)."""
    cases = [("int2_sym", 64, 5), ("fp8_e5m2", 32, 12), ("int2_sym", 32, 70),
             ("fp8_e5m2", 256, 200)]
    N, K = 128, 1024
    prepared = []
    for fmt, G, M in cases:
        W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=68)
        pw = wq.pack(fmt, N, K, G, dev_u8(codes), dev_u8(scales), None)
        x = synth.activations(69, M, K)
        ref, _ = orc.linear(x, orc.dequant(fmt, codes, scales, aux, N, K, G), None)
        prepared.append((pw, x, ref, M))
    results, errors = [None] * len(cases), []

    def work(i):
        try:
            pw, x, ref, M = prepared[i]
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                xd = dev_bf16(x)
                y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
                wq.wq_linear(xd, pw.w, pw.scales, pw.aux, None, M, N, K, pw.fmt, pw.group_size,
                             y, s)
            s.synchronize()
            results[i] = bf16_bits(y)
        except Exception as e:  # noqa: BLE001 - reported below
            errors.append(repr(e))

    ts = [threading.Thread(target=work, args=(i,)) for i in range(len(cases))]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors
    for (pw, x, ref, M), y in zip(prepared, results):
        check_close(y, ref, f"{pw.fmt} M={M} from a thread")
