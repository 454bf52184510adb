"""GPU LoRA merge into a packed INT8 weight, code for code against the oracle
(nearest and seeded stochastic requantization; rank 0 is a no-op; other
formats are refused)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_cases import dev_bf16, pack_on_gpu, small_case

pytestmark = pytest.mark.gpu


def _unpack_codes(wq, pw, N, K, G):
    cb, cs, _ = wq.wq_canonical_sizes("int8_sym", N, K, G)
    c = torch.zeros(cb, dtype=torch.uint8, device="cuda")
    s = torch.zeros(cs, dtype=torch.uint8, device="cuda")
    wq.wq_unpack("int8_sym", N, K, G, pw.w, pw.scales, pw.aux, c, s, None)
    torch.cuda.synchronize()
    return c.cpu().numpy().view(np.int8).reshape(N, K)


@pytest.mark.parametrize("G", [64, 256])
@pytest.mark.parametrize("seed", [None, 2024])
def test_addmm_requant_matches_oracle(wq, orc, G, seed):
    N, K, R = 96, 1024, 16
    W, (codes, scales, _) = small_case(orc, "int8_sym", N, K, G, seed=21)
    pw = pack_on_gpu(wq, "int8_sym", N, K, G, codes, scales, None)
    m1 = synth.activations(31, N, R, sigma=0.05)          # lora_b [N, R]
    m2 = synth.activations(32, R, K, sigma=0.05)          # lora_a [R, K]
    alpha, beta = 0.75, 1.0
    wq.wq_addmm_requant("int8_sym", N, K, G, pw.w, pw.scales, dev_bf16(m1), dev_bf16(m2), R,
                        alpha, beta, seed)
    got = _unpack_codes(wq, pw, N, K, G)
    want = orc.addmm_requant_int8(codes, scales, G, m1, m2, alpha, beta, seed)
    assert np.array_equal(got, want)
    assert not np.array_equal(want, codes)                # the update moved some codes


def test_addmm_requant_noop_and_unsupported(wq, orc):
    N, K, G = 32, 256, 64
    W, (codes, scales, _) = small_case(orc, "int8_sym", N, K, G, seed=22)
    pw = pack_on_gpu(wq, "int8_sym", N, K, G, codes, scales, None)
    wq.wq_addmm_requant("int8_sym", N, K, G, pw.w, pw.scales, None, None, 0, 1.0, 1.0)
    assert np.array_equal(_unpack_codes(wq, pw, N, K, G), codes)
    W4, (c4, s4, _) = small_case(orc, "int4_sym", N, K, G, seed=23)
    pw4 = pack_on_gpu(wq, "int4_sym", N, K, G, c4, s4, None)
    with pytest.raises(wq.WQError) as ei:
        wq.wq_addmm_requant("int4_sym", N, K, G, pw4.w, pw4.scales, None, None, 0, 1.0, 1.0)
    assert ei.value.status == wq.WQ_ERR_UNSUPPORTED
