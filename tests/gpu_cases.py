"""Helpers for the GPU parity tests: inputs from the seeded generator, expected
values from the oracle, device buffers through torch, calls through the
C-ABI binding."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

TOL_REL = 1e-2  # |y - y_ref| <= 1e-2 * max(1, |y_ref|), y_ref = bf16(fp64 result)


def dev_u8(a: np.ndarray) -> torch.Tensor:
    """numpy array -> flat uint8 CUDA tensor holding the same bytes (>= 16 bytes)."""
    b = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
    t = torch.zeros((max(b.size, 16),), dtype=torch.uint8, device="cuda")
    t[: b.size].copy_(torch.from_numpy(b.copy()))
    return t


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(
        torch.bfloat16).cuda()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def canonical(orc, fmt, W, G):
    codes, scales, aux = orc.quantize(fmt, W, G)
    return codes, scales, aux


def pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux):
    cb, cs, ca = wq.wq_canonical_sizes(fmt, N, K, G)
    assert cb == codes.nbytes and cs == scales.nbytes
    return wq.pack(fmt, N, K, G, dev_u8(codes), dev_u8(scales),
                   dev_u8(aux) if aux is not None else None)


def check_close(y_bits: np.ndarray, ref_bits: np.ndarray, what: str = ""):
    y = oracle.bits_to_f32(y_bits).astype(np.float64)
    r = oracle.bits_to_f32(ref_bits).astype(np.float64)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.abs(y - r)
    lim = TOL_REL * np.maximum(1.0, np.abs(r))
    bad = err > lim
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at "
                             f"{tuple(i)}: got {y[tuple(i)]} want {r[tuple(i)]}")
    return float((err / lim).max()) if err.size else 0.0


GUARD_BEFORE = 128    # bf16 elements (256 bytes: the output stays 16-byte aligned)
GUARD_AFTER = 4096    # bf16 elements
GUARD_BITS = 0x7FA5   # a NaN pattern no kernel writes


def guarded_out(M: int, N: int) -> tuple[torch.Tensor, torch.Tensor]:
    """(buffer, out): ``out`` is an [M, N] bf16 view inside ``buffer`` with
    canary bands before and after it; the output itself starts as NaN, so an
    element the kernel never writes is caught as non-finite."""
    buf = torch.full((GUARD_BEFORE + max(M, 1) * N + GUARD_AFTER,), GUARD_BITS, dtype=torch.int16,
                     device="cuda")
    out = buf[GUARD_BEFORE:GUARD_BEFORE + max(M, 1) * N].view(torch.bfloat16).view(max(M, 1), N)
    out.fill_(float("nan"))
    return buf, out


def check_guards(buf: torch.Tensor, M: int, N: int, what: str = ""):
    """Both canary bands around a guarded output are untouched."""
    b = buf.cpu().numpy().view(np.uint16)
    head, tail = b[:GUARD_BEFORE], b[GUARD_BEFORE + max(M, 1) * N:]
    assert np.all(head == GUARD_BITS), f"{what}: write before the output ({np.sum(head != GUARD_BITS)})"
    assert np.all(tail == GUARD_BITS), f"{what}: write past the output ({np.sum(tail != GUARD_BITS)})"


def run_linear(wq, pw, x_bits, bias_bits, M, stream=None):
    """One wq_linear call through the C ABI into a guarded output buffer; the
    canaries around the output are checked before the result is returned."""
    x = dev_bf16(x_bits)
    b = dev_bf16(bias_bits) if bias_bits is not None else None
    buf, y = guarded_out(M, pw.N)
    wq.wq_linear(x, pw.w, pw.scales, pw.aux, b, M, pw.N, pw.K, pw.fmt, pw.group_size, y, stream)
    torch.cuda.synchronize()
    check_guards(buf, M, pw.N, f"{pw.fmt} M={M} N={pw.N} K={pw.K}")
    return bf16_bits(y[:M])


def small_case(orc, fmt, N, K, G, seed, dist="normal"):
    W = synth.weight(seed, N, K, dist=dist, sigma=0.02, outlier_count=(N * K) // 1000,
                     outlier_mult=20.0)
    return W, canonical(orc, fmt, W, G)
