"""GPU parity at the seven workloads' full sizes, in the launch configuration
the benchmark times (the same wq_linear call).  Small batches are compared
element by element against the full oracle product; large ones on sampled
outputs that the oracle computes one by one.  The GPU quantizer (which the
benchmark uses to make its inputs) is checked bit for bit against the
oracle's quantizer at full size."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth.workloads as W
from gpu_cases import check_close, dev_bf16, dev_u8, pack_on_gpu, run_linear

pytestmark = pytest.mark.gpu

_cache = {}


def _workload(orc, wq, wl):
    if wl.name in _cache:
        return _cache[wl.name]
    Wd = W.make_weight(wl)
    G = wl.group_size
    codes, scales, aux = orc.quantize(wl.fmt, Wd, G)
    pw = pack_on_gpu(wq, wl.fmt, wl.N, wl.K, G, codes, scales, aux)
    # GPU quantizer on the same dense weight, compared byte for byte
    cb, cs, ca = wq.wq_canonical_sizes(wl.fmt, wl.N, wl.K, G)
    dc = torch.zeros(cb, dtype=torch.uint8, device="cuda")
    ds = torch.zeros(cs, dtype=torch.uint8, device="cuda")
    da = torch.zeros(max(ca, 16), dtype=torch.uint8, device="cuda") if ca else None
    if wl.fmt == "cb4":
        da.view(torch.float32)[:16].copy_(torch.from_numpy(wq.wq_lloyd_max_centroids(4)))
    wd = torch.from_numpy(Wd).cuda()
    wq.wq_quantize(wl.fmt, wl.N, wl.K, G, wd, dc, ds, da)
    torch.cuda.synchronize()
    same = (np.array_equal(dc.cpu().numpy(), codes.view(np.uint8).reshape(-1))
            and np.array_equal(ds.cpu().numpy(), scales.view(np.uint8).reshape(-1))
            and (not ca or np.array_equal(da[:ca].cpu().numpy(), aux.view(np.uint8).reshape(-1))))
    del wd, dc, ds, da
    xa = W.make_x(wl, max(wl.Ms))
    b = W.make_bias(wl)
    _cache.clear()
    _cache[wl.name] = (codes, scales, aux, pw, xa, b, same)
    return _cache[wl.name]


def _samples(M, N, count, seed):
    rng = np.random.default_rng(seed)
    ms = rng.integers(0, M, count)
    ns = rng.integers(0, N, count)
    # edges: first / last token and feature
    ms = np.concatenate([ms, [0, 0, M - 1, M - 1]])
    ns = np.concatenate([ns, [0, N - 1, 0, N - 1]])
    return ms, ns


@pytest.mark.parametrize("wl", W.ALL, ids=[w.name for w in W.ALL])
def test_workload_parity(wq, orc, wl):
    codes, scales, aux, pw, xa, b, same = _workload(orc, wq, wl)
    assert same, "GPU quantizer differs from the oracle's at full size"
    G = wl.group_size
    full_limit = 2_000_000_000  # multiply-adds the oracle does in full
    dq = None
    for M in wl.Ms:
        y = run_linear(wq, pw, xa[:M], b, M)
        assert y.shape == (M, wl.N)
        assert np.all(np.isfinite(y.view(np.int16).astype(np.float32)))
        if M * wl.N * wl.K <= full_limit:
            if dq is None:
                dq = orc.dequant(wl.fmt, codes, scales, aux, wl.N, wl.K, G)
            ref, _ = orc.linear(xa[:M], dq, b)
            check_close(y, ref, f"{wl.name} M={M}")
        else:
            ms, ns = _samples(M, wl.N, 1500, seed=M)
            ref, _ = orc.linear_sampled(wl.fmt, codes, scales, aux, wl.N, wl.K, G, xa[:M], b,
                                        ms, ns)
            check_close(y[ms, ns], ref, f"{wl.name} M={M} (sampled)")
            # a whole output row and a whole output column as well
            rows = np.zeros(wl.N, np.int64) + (M // 2)
            cols = np.arange(wl.N)
            rref, _ = orc.linear_sampled(wl.fmt, codes, scales, aux, wl.N, wl.K, G, xa[:M], b,
                                         rows, cols)
            check_close(y[M // 2], rref, f"{wl.name} M={M} row {M // 2}")
