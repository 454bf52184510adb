"""User-facing helpers over the C ABI: a packed weight handle and ``linear``.

torch provides device memory and streams only; quantization, packing and the
linear itself run in ``libwq.so``.  This mirrors the reference APIs: a dense
weight is quantized and repacked once (piper-kernels ``from_hp``,
auto-round-lib ``repack_quantized_weight``), then used as a linear weight
(``F.linear`` / ``woqgemm`` / ``matmul_packed_weight``).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (FORMATS, wq_canonical_sizes, wq_linear, wq_linear_a8, wq_linear_a8_workspace_size,
               wq_linear_grouped, wq_linear_grouped_dev, wq_linear_swiglu,
               wq_lloyd_max_centroids, wq_pack, wq_packed_sizes, wq_quantize)


@dataclass
class PackedWeight:
    """Packed buffers of one [N, K] weight (or, with ``experts`` > 1, of
    that many experts' weights stacked back to back), on a CUDA device."""
    fmt: str
    N: int
    K: int
    group_size: int
    w: torch.Tensor        # packed codes (uint8)
    scales: torch.Tensor   # packed scales (uint8 view of the bytes)
    aux: torch.Tensor | None
    experts: int = 1

    @property
    def nbytes(self) -> int:
        return self.w.numel() + self.scales.numel() + (0 if self.aux is None else self.aux.numel())

    def clone(self) -> "PackedWeight":
        c = PackedWeight(self.fmt, self.N, self.K, self.group_size, self.w.clone(),
                         self.scales.clone(), None if self.aux is None else self.aux.clone(),
                         self.experts)
        torch.cuda.synchronize(self.w.device)  # final before any wq_linear prefetches it
        return c


def _bytes(n: int, device) -> torch.Tensor:
    # at least 16 bytes so every buffer has a valid, aligned address
    return torch.empty((max(int(n), 16),), dtype=torch.uint8, device=device)


def pack(fmt: str, N: int, K: int, group_size: int, codes: torch.Tensor, scales: torch.Tensor,
         aux: torch.Tensor | None, stream=None) -> PackedWeight:
    """Canonical device buffers -> PackedWeight (wq_pack).

    Offline: waits for the pack to finish, so that the packed buffers are
    final before any wq_linear that may prefetch them (see wq.h)."""
    dev = codes.device
    wb, sb, ab = wq_packed_sizes(fmt, N, K, group_size)
    pw, ps = _bytes(wb, dev), _bytes(sb, dev)
    pa = _bytes(ab, dev) if ab else None
    wq_pack(fmt, N, K, group_size, codes, scales, aux, pw, ps, pa, stream)
    torch.cuda.synchronize(dev)
    return PackedWeight(fmt, N, K, group_size, pw, ps, pa)


def quantize_and_pack(w: torch.Tensor, fmt: str, group_size: int = 0, centroids=None,
                      stream=None) -> PackedWeight:
    """Dense fp32 [N, K] device weight -> round-to-nearest quantized PackedWeight.

    For ``cb4`` the 16 centroids default to the Lloyd-Max quantizer of N(0,1).
    """
    assert w.is_cuda and w.dtype == torch.float32 and w.is_contiguous()
    N, K = w.shape
    dev = w.device
    cb, sb, ab = wq_canonical_sizes(fmt, N, K, group_size)
    codes, scales = _bytes(cb, dev), _bytes(sb, dev)
    aux = _bytes(ab, dev) if ab else None
    if fmt == "cb4":
        c = wq_lloyd_max_centroids(4) if centroids is None else centroids
        aux.view(torch.float32)[:16].copy_(torch.as_tensor(c, dtype=torch.float32))
    wq_quantize(fmt, N, K, group_size, w, codes, scales, aux, stream)
    return pack(fmt, N, K, group_size, codes, scales, aux, stream)


def _torch_stream(stream, dev) -> torch.cuda.Stream:
    """The torch stream object for ``stream`` (None: the device's current
    stream; an integer: an existing cudaStream_t)."""
    if stream is None:
        return torch.cuda.current_stream(dev)
    if isinstance(stream, int):
        return torch.cuda.ExternalStream(stream, device=dev)
    return stream


def linear(x: torch.Tensor, weight: PackedWeight, bias: torch.Tensor | None = None,
           out: torch.Tensor | None = None, stream=None, sync: bool = True) -> torch.Tensor:
    """y = x @ dequant(weight).T + bias, bf16.  ``x``: [..., K] bf16.

    A host (CPU) ``x`` is copied to the weight's device and the result copied
    back, so the call works end to end from host memory; both copies and the
    linear run in order on ``stream`` (default: the current stream).  With a
    host ``x`` and ``sync=False`` the copy back is only enqueued (into
    ``out``, which should then be pinned host memory): synchronize the stream
    before reading it, e.g. once after several calls.
    """
    host = not x.is_cuda
    dev = weight.w.device
    lead = x.shape[:-1]
    K = x.shape[-1]
    assert K == weight.K and x.dtype == torch.bfloat16
    s = _torch_stream(stream, dev)
    with torch.cuda.stream(s):
        xd = x.reshape(-1, K)
        if host:
            xd = xd.to(dev, non_blocking=True)
        xd = xd.contiguous()
        M = xd.shape[0]
        if bias is not None and not bias.is_cuda:
            bias = bias.to(dev, non_blocking=True)
        y = out if (out is not None and not host) else torch.empty(
            (M, weight.N), dtype=torch.bfloat16, device=dev)
        wq_linear(xd, weight.w, weight.scales, weight.aux, bias, M, weight.N, K, weight.fmt,
                  weight.group_size, y, s)
        if host:
            yh = out if out is not None else torch.empty((M, weight.N), dtype=torch.bfloat16,
                                                          pin_memory=True)
            yh.copy_(y, non_blocking=True)
    if host:
        if sync:
            s.synchronize()
        return yh.reshape(*lead, weight.N)
    return y.reshape(*lead, weight.N)


def linear_swiglu(x2: torch.Tensor, weight: PackedWeight, bias: torch.Tensor | None = None,
                  out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = (up * silu(gate)) @ dequant(weight).T + bias for ``x2`` = [..., 2K] =
    [up | gate] (bf16, on the weight's device).  For more than 16 rows the
    activation is materialized in a torch-allocated workspace."""
    dev = weight.w.device
    lead = x2.shape[:-1]
    K = weight.K
    assert x2.shape[-1] == 2 * K and x2.dtype == torch.bfloat16 and x2.is_cuda
    xd = x2.reshape(-1, 2 * K).contiguous()
    M = xd.shape[0]
    y = out if out is not None else torch.empty((M, weight.N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if M > 16 else None
    wq_linear_swiglu(xd, weight.w, weight.scales, weight.aux, bias, M, weight.N, K, weight.fmt,
                     weight.group_size, ws, 0 if ws is None else ws.numel() * 2, y, stream)
    return y.reshape(*lead, weight.N)


def linear_a8(x: torch.Tensor, weight: PackedWeight, bias: torch.Tensor | None = None,
              out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
              stream=None, sync: bool = True) -> torch.Tensor:
    """Activation-quantized linear (INT8 weights): x quantized per token to
    INT8, integer tensor-core products, group scales and the token scale
    applied in fp32.  ``x``: [..., K] bf16.  The INT8 activations live in
    ``workspace`` (allocated here when not given).  A host ``x`` is copied in
    and the result copied back on ``stream``, as in ``linear``."""
    host = not x.is_cuda
    dev = weight.w.device
    lead = x.shape[:-1]
    K = weight.K
    assert x.shape[-1] == K and x.dtype == torch.bfloat16
    s = _torch_stream(stream, dev)
    with torch.cuda.stream(s):
        xd = x.reshape(-1, K)
        if host:
            xd = xd.to(dev, non_blocking=True)
        xd = xd.contiguous()
        M = xd.shape[0]
        need = wq_linear_a8_workspace_size(M, K)
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=dev)
        y = out if (out is not None and not host) else torch.empty(
            (M, weight.N), dtype=torch.bfloat16, device=dev)
        wq_linear_a8(xd, weight.w, weight.scales, bias, M, weight.N, K, weight.fmt,
                     weight.group_size, workspace, workspace.numel() * workspace.element_size(),
                     y, s)
        if host:
            yh = out if out is not None else torch.empty((M, weight.N), dtype=torch.bfloat16,
                                                          pin_memory=True)
            yh.copy_(y, non_blocking=True)
    if host:
        if sync:
            s.synchronize()
        return yh.reshape(*lead, weight.N)
    return y.reshape(*lead, weight.N)


def stack_experts(weights: list) -> PackedWeight:
    """E PackedWeights of one format, shape and group size -> one PackedWeight
    whose buffers hold them back to back at the packed sizes (the layout
    ``linear_moe`` and wq_linear_grouped_dev read)."""
    w0 = weights[0]
    assert all(w.fmt == w0.fmt and w.N == w0.N and w.K == w0.K and
               w.group_size == w0.group_size and w.experts == 1 for w in weights)
    wb, sb, ab = wq_packed_sizes(w0.fmt, w0.N, w0.K, w0.group_size)
    cat = lambda ts, n: torch.cat([t[:n] for t in ts] + [torch.zeros(16, dtype=torch.uint8,
                                                                     device=ts[0].device)])
    aux = cat([w.aux for w in weights], ab) if ab else None
    return PackedWeight(w0.fmt, w0.N, w0.K, w0.group_size, cat([w.w for w in weights], wb),
                        cat([w.scales for w in weights], sb), aux, experts=len(weights))


def linear_moe(x: torch.Tensor, experts: PackedWeight, offsets: torch.Tensor,
               bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """Mixture-of-experts linear in one launch with device-side routing:
    rows offsets[e]:offsets[e+1] of ``x`` ([T, K] bf16, sorted by expert) use
    expert e of ``experts`` (from ``stack_experts``); ``offsets`` is a device
    int64 tensor [E + 1] (e.g. a cumulative sum of a router's counts);
    ``bias`` an optional [E, N] bf16 tensor.  Rows no expert owns are left
    as they are in ``out``."""
    E = experts.experts
    assert offsets.is_cuda and offsets.dtype == torch.int64 and offsets.numel() == E + 1
    xd = x.contiguous()
    T = xd.shape[0]
    assert xd.shape == (T, experts.K)
    y = out if out is not None else torch.zeros((T, experts.N), dtype=torch.bfloat16,
                                                device=experts.w.device)
    wq_linear_grouped_dev(xd, experts.w, experts.scales, experts.aux, bias, offsets.contiguous(),
                          E, T, experts.N, experts.K, experts.fmt, experts.group_size, y, stream)
    return y


def linear_grouped(x: torch.Tensor, weights: list, offsets, bias: list | None = None,
                   out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Mixture-of-experts linear: rows offsets[e]:offsets[e+1] of ``x`` ([T, K]
    bf16, sorted by expert) use ``weights[e]`` (PackedWeights of one format,
    shape and group size); ``bias`` an optional list of per-expert [N] tensors."""
    w0 = weights[0]
    assert all(w.fmt == w0.fmt and w.N == w0.N and w.K == w0.K and
               w.group_size == w0.group_size for w in weights)
    xd = x.contiguous()
    T = int(offsets[-1])
    assert xd.shape == (T, w0.K) and len(offsets) == len(weights) + 1
    y = out if out is not None else torch.empty((T, w0.N), dtype=torch.bfloat16,
                                                device=w0.w.device)
    wq_linear_grouped(xd, [w.w for w in weights], [w.scales for w in weights],
                      None if w0.aux is None else [w.aux for w in weights], bias,
                      [int(o) for o in offsets], w0.N, w0.K, w0.fmt, w0.group_size, y, stream)
    return y
