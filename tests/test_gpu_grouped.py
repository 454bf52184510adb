"""GPU parity of the grouped (mixture-of-experts) linear: experts of one
format with per-expert row counts (an empty expert, decode-sized and
prefill-sized slices), each slice against the oracle with that expert's
weight."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_cases import bf16_bits, check_close, dev_bf16, pack_on_gpu, small_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,G", [("int4_asym", 128), ("nvfp4", 16), ("fp8_e4m3", 64)])
def test_grouped_matches_per_expert_oracle(wq, orc, fmt, G):
    N, K = 96, 512
    counts = [0, 3, 40, 1, 17]
    offsets = np.concatenate([[0], np.cumsum(counts)])
    T = int(offsets[-1])
    experts, dqs, biases = [], [], []
    for e in range(len(counts)):
        W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=100 + e)
        experts.append(pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux))
        dqs.append(orc.dequant(fmt, codes, scales, aux, N, K, G))
        biases.append(synth.bias(200 + e, N))
    xa = synth.activations(71, T, K)
    for with_bias in (False, True):
        bias = [dev_bf16(b) for b in biases] if with_bias else None
        y = wq.linear_grouped(dev_bf16(xa), experts, offsets, bias=bias)
        torch.cuda.synchronize()
        yb = bf16_bits(y)
        for e in range(len(counts)):
            a, b = int(offsets[e]), int(offsets[e + 1])
            if a == b:
                continue
            ref, _ = orc.linear(xa[a:b], dqs[e], biases[e] if with_bias else None)
            check_close(yb[a:b], ref, f"{fmt} expert {e} bias={with_bias}")
