"""GPU parity at the seven workloads' full sizes, in the launch configuration
the benchmark times (the same wq_linear call).  Every batch size of every
workload is compared element by element against the oracle's full product
(its fp64 library-matmul form, seconds even for the 4096 x 8192 x 8192
prefill case), and canary bands around each output are checked untouched.
The GPU quantizer (which the benchmark uses to make its inputs) is checked
bit for bit against the oracle's quantizer at full size."""
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


@pytest.mark.parametrize("wl", W.ALL, ids=[w.name for w in W.ALL])
def test_workload_parity(wq, orc, wl):
    codes, scales, aux, pw, xa, b, same = _workload(orc, wq, wl)
    assert same, "GPU quantizer differs from the oracle's at full size"
    G = wl.group_size
    dq = orc.dequant(wl.fmt, codes, scales, aux, wl.N, wl.K, G)
    for M in wl.Ms:
        y = run_linear(wq, pw, xa[:M], b, M)
        assert y.shape == (M, wl.N)
        ref, _ = orc.linear_full(xa[:M], dq, b)
        check_close(y, ref, f"{wl.name} M={M}")
