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


def _experts(wq, orc, fmt, G, N, K, E, seed0):
    packed, dqs = [], []
    for e in range(E):
        W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=seed0 + e)
        packed.append(pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux))
        dqs.append(orc.dequant(fmt, codes, scales, aux, N, K, G))
    return wq.stack_experts(packed), dqs


def _skewed_counts(E, T, seed):
    """Per-expert row counts summing to T, Zipf-like skew, several experts empty."""
    rng = np.random.default_rng(seed)
    w = 1.0 / np.arange(1, E + 1) ** 1.1
    w = w[rng.permutation(E)]
    c = rng.multinomial(T, w / w.sum()).astype(np.int64)
    for e in (3, 17, E - 1):                        # a few experts always empty
        c[0] += c[e]
        c[e] = 0
    return c


@pytest.mark.parametrize("fmt,G,T", [("int4_asym", 128, 3000), ("int4_asym", 128, 40),
                                     ("nvfp4", 16, 700), ("int8_sym", 256, 1500),
                                     ("cb4", 0, 300), ("mxfp4", 32, 64),
                                     ("fp8_e4m3", 64, 500), ("int2_sym", 64, 900)])
def test_one_launch_grouped_matches_per_expert_oracle(wq, orc, fmt, G, T):
    """wq_linear_grouped_dev: 64 experts, skewed device-resident counts (many
    experts empty at T = 40), every owned output against the oracle with that
    expert's weight; canary rows past the last expert stay untouched."""
    E, N, K = 64, 256, 512
    experts, dqs = _experts(wq, orc, fmt, G, N, K, E, seed0=300)
    counts = _skewed_counts(E, T, seed=T)
    assert (counts == 0).any()
    offsets = np.concatenate([[0], np.cumsum(counts)])
    extra = 5                                               # rows no expert owns
    xa = synth.activations(81, T + extra, K)
    bias = np.stack([synth.bias(400 + e, N) for e in range(E)])
    for with_bias in (False, True):
        y = torch.full((T + extra, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        off_d = torch.from_numpy(offsets).cuda()
        wq.linear_moe(dev_bf16(xa), experts, off_d, bias=dev_bf16(bias) if with_bias else None,
                      out=y)
        torch.cuda.synchronize()
        assert wq.wq_device_error() == 0
        yb = bf16_bits(y)
        assert np.all(yb[T:] == 0x7FC0)                      # not owned: not written
        for e in range(E):
            a, b = int(offsets[e]), int(offsets[e + 1])
            if a == b:
                continue
            ref, _ = orc.linear_full(xa[a:b], dqs[e], bias[e] if with_bias else None)
            check_close(yb[a:b], ref, f"{fmt} expert {e} ({b - a} rows) bias={with_bias}")


def test_one_launch_grouped_bad_offsets(wq, orc):
    """A decreasing or out-of-range offset makes its expert empty (nothing
    written for it) and raises bit 256 of the device error word; the other
    experts are still computed."""
    E, N, K, G = 4, 128, 256, 64
    experts, dqs = _experts(wq, orc, "int4_sym", G, N, K, E, seed0=500)
    T = 40
    offsets = np.array([0, 10, 5, 30, 90], np.int64)   # expert 1 decreasing, expert 3 past T
    xa = synth.activations(82, T, K)
    y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    wq.linear_moe(dev_bf16(xa), experts, torch.from_numpy(offsets).cuda(), out=y)
    torch.cuda.synchronize()
    assert wq.wq_device_error() & 256
    assert wq.wq_device_error() == 0                         # read-and-clear
    yb = bf16_bits(y)
    ref0, _ = orc.linear_full(xa[0:10], dqs[0], None)
    check_close(yb[0:5], ref0[:5], "expert 0 (rows 0..4; rows 5..9 are also expert 2's)")
    ref2, _ = orc.linear_full(xa[5:30], dqs[2], None)
    check_close(yb[10:30], ref2[5:], "expert 2 (rows 10..29)")
    assert np.all(yb[30:] == 0x7FC0)
