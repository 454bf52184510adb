"""GPU parity where the tcgen05 kernel's persistent CTAs take several tiles
each (more tiles than SMs) and the last token tile is ragged: one linear of
N = 9216 (72 column blocks) at M = 777 (four token tiles of 256, the last
with 9 rows), K = 1024, in three formats, compared element by element with
the oracle's full product; and the same through the grouped launch, whose
persistent CTAs look their tiles up in the device-side schedule, with
ragged expert counts."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_cases import check_close, dev_bf16, pack_on_gpu, run_linear, small_case

pytestmark = pytest.mark.gpu

N, K, M = 9216, 1024, 777


@pytest.mark.parametrize("fmt,G", [("int8_sym", 256), ("int4_asym", 128), ("nvfp4", 16)])
def test_multi_tile_ragged(wq, orc, fmt, G):
    sms = wq.wq_device_sm_count()
    tiles = (N // 128) * -(-M // 256)
    assert tiles > sms, "the case must give some CTAs more than one tile"
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=41)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    x = synth.activations(42, M, K)
    b = synth.bias(43, N)
    y = run_linear(wq, pw, x, b, M)
    dq = orc.dequant(fmt, codes, scales, aux, N, K, G)
    ref, _ = orc.linear_full(x, dq, b)
    check_close(y, ref, f"{fmt} N={N} K={K} M={M}")


def test_grouped_many_tiles(wq, orc):
    """16 INT4 experts of 2048 x 512 with ragged counts (one empty): the
    grouped launch's persistent CTAs take several schedule tiles each."""
    import mixed_gemm_b200.api as api
    E, Ne, Ke, G = 16, 2048, 512, 128
    rng = np.random.default_rng(5)
    counts = rng.integers(200, 700, size=E)
    counts[3] = 0
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    T = int(offs[-1])
    tiles = (Ne // 128) * int(sum(-(-c // 256) for c in counts))
    assert tiles > wq.wq_device_sm_count()
    pws, dqs = [], []
    for e in range(E):
        W, (codes, scales, aux) = small_case(orc, "int4_sym", Ne, Ke, G, seed=100 + e)
        pws.append(pack_on_gpu(wq, "int4_sym", Ne, Ke, G, codes, scales, aux))
        dqs.append(orc.dequant("int4_sym", codes, scales, aux, Ne, Ke, G))
    ex = api.stack_experts(pws)
    x = synth.activations(44, T, Ke)
    xd = dev_bf16(x)
    out = torch.full((T, Ne), float("nan"), dtype=torch.bfloat16, device="cuda")
    api.linear_moe(xd, ex, torch.from_numpy(offs).cuda(), out=out)
    torch.cuda.synchronize()
    y = out.cpu().view(torch.int16).numpy().view(np.uint16)
    for e in range(E):
        a, c = int(offs[e]), int(offs[e + 1])
        if c == a:
            continue
        ref, _ = orc.linear_full(x[a:c], dqs[e], None)
        check_close(y[a:c], ref, f"expert {e} rows {c - a}")
