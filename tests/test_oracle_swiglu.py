"""Pins of the oracle's SwiGLU input step (piper-kernels README: the SwiGLU
input [..., 2K] = [up | gate] is turned into up * silu(gate) before the
linear): silu against torch's own silu in fp64 and its closed-form
properties; the bf16 activation against an independent rounding."""
from __future__ import annotations

import math

import numpy as np
import torch

import synth


def test_silu_matches_torch_and_identities(orc):
    g = np.concatenate([np.linspace(-40, 40, 2001), [0.0, 1e-300, -1e-300, 700.0, -700.0]])
    ref = torch.nn.functional.silu(torch.from_numpy(g)).numpy()
    got = np.array([orc.silu(float(v)) for v in g])
    assert np.allclose(got, ref, rtol=1e-14, atol=1e-300)
    assert orc.silu(0.0) == 0.0
    # silu(g) - silu(-g) = g  (g * (sigma(g) + sigma(-g)) = g)
    for v in (0.3, 1.7, 5.0, 13.0):
        assert math.isclose(orc.silu(v) - orc.silu(-v), v, rel_tol=1e-14)
    assert orc.silu(700.0) == 700.0 and abs(orc.silu(-700.0)) < 1e-290


def test_swiglu_layout_and_rounding(orc):
    M, K = 5, 96
    x2 = synth.activations(3, M, 2 * K)
    a = orc.swiglu(x2)
    assert a.shape == (M, K)
    def val(bits):  # bf16 bits -> value: the high half of an fp32
        return (np.ascontiguousarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    up = val(x2[:, :K])
    gate = val(x2[:, K:])
    want = synth.f64_to_bf16_bits(
        up * torch.nn.functional.silu(torch.from_numpy(gate)).numpy())
    assert np.array_equal(a, want)
    # up and gate are not interchangeable
    swapped = synth.f64_to_bf16_bits(
        gate * torch.nn.functional.silu(torch.from_numpy(up)).numpy())
    assert not np.array_equal(a, swapped)
