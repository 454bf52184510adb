"""The seven synthetic workloads of the weight-only quantized linear.

Each recipe fixes shapes, the weight format, the group size, the seed and the
value distributions; ``make_inputs`` draws the dense inputs for one of them.
Format names are the library's: int4_sym, int4_asym, int8_sym, cb4, nvfp4, mxfp4,
fp8_e4m3.

Readings (the recipe texts leave these open):
  * seeds other than the first workload's are 1, 2, 3, 4 in order, and 5
    for the MXFP4 twin of the NVFP4 shape (same layer, same distribution),
    6 for the FP8 E4M3 weight-only layer (the INT8 prefill layer's shape and
    distribution, group 128, decode and prefill batch sizes);
  * "0.1% of entries replaced by x20 outliers" = round(0.001*N*K) distinct
    positions whose drawn value is multiplied by 20;
  * "1% of channels scaled x10" = round(0.01*K) distinct input columns of X
    multiplied by 10;
  * a bias whose sigma is not given reuses N(0, 0.01^2); a workload that does
    not mention a bias has none.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import activations, bias as draw_bias, weight


@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str
    N: int
    K: int
    Ms: tuple
    group_size: int
    seed: int
    w_dist: str = "normal"
    w_sigma: float = 0.02
    w_outlier_frac: float = 0.0
    w_outlier_mult: float = 1.0
    x_channel_frac: float = 0.0
    x_channel_mult: float = 1.0
    bias_sigma: float | None = None
    note: str = ""
    act_int8: bool = False   # activation-quantized linear (per-token INT8 x)

    @property
    def w_outlier_count(self) -> int:
        return int(round(self.w_outlier_frac * self.N * self.K))

    @property
    def x_channel_count(self) -> int:
        return int(round(self.x_channel_frac * self.K))


PR1 = Workload("pr1_int4_sym_g64", "int4_sym", N=256, K=512, Ms=(4,), group_size=64, seed=0,
               bias_sigma=0.01, note="first slice: INT4 sym g64, M=4")
DECODE = Workload("decode_int4_asym_g128", "int4_asym", N=4096, K=4096, Ms=(1, 2, 4, 8, 16),
                  group_size=128, seed=1, w_outlier_frac=0.001, w_outlier_mult=20.0,
                  note="decode sweep on a 4096x4096 layer, asym INT4 + uint4 zero-point")
CODEBOOK = Workload("codebook4_3072", "cb4", N=3072, K=3072, Ms=(1, 16, 256), group_size=0,
                    seed=2, bias_sigma=0.01, note="4-bit Lloyd-Max codebook with row norms")
NVFP4 = Workload("nvfp4_28672x8192", "nvfp4", N=28672, K=8192, Ms=(1, 8, 64, 256),
                 group_size=16, seed=3, w_dist="student5",
                 note="NVFP4 70B-class MLP up-projection shape")
MXFP4 = Workload("mxfp4_28672x8192", "mxfp4", N=28672, K=8192, Ms=(1, 8, 64, 256),
                 group_size=32, seed=5, w_dist="student5",
                 note="MXFP4 (E8M0 scale per 32) on the NVFP4 layer shape")
PREFILL = Workload("prefill_int8_g256", "int8_sym", N=8192, K=8192, Ms=(1024, 2048, 4096),
                   group_size=256, seed=4, x_channel_frac=0.01, x_channel_mult=10.0,
                   bias_sigma=0.01, note="compute-bound prefill, INT8 sym g256")

FP8 = Workload("fp8_e4m3_8192", "fp8_e4m3", N=8192, K=8192, Ms=(1, 16, 1024), group_size=128,
               seed=6, note="FP8 E4M3 weight-only, fp32 scale per 128 along K")
INT3 = Workload("int3_sym_g128_8192", "int3_sym", N=8192, K=8192, Ms=(1, 16, 1024),
                group_size=128, seed=9, note="INT3 sym g128 (two-plane packed layout)")

# the prefill layer and inputs again, through the activation-quantized linear
A8 = Workload("a8_int8_g256_8192", "int8_sym", N=8192, K=8192, Ms=(1024, 2048, 4096),
              group_size=256, seed=4, x_channel_frac=0.01, x_channel_mult=10.0,
              bias_sigma=0.01, act_int8=True,
              note="W8A8: the prefill layer with per-token INT8 activations")

ALL = (PR1, DECODE, CODEBOOK, NVFP4, PREFILL, MXFP4, FP8, INT3)
BY_NAME = {w.name: w for w in ALL + (A8,)}


def make_weight(w: Workload) -> np.ndarray:
    return weight(w.seed, w.N, w.K, dist=w.w_dist, sigma=w.w_sigma,
                  outlier_count=w.w_outlier_count, outlier_mult=w.w_outlier_mult)


def make_x(w: Workload, M: int) -> np.ndarray:
    """X[M, K] bf16 bits.  Row m is the same for every M (one stream per workload)."""
    return activations(w.seed, M, w.K, sigma=1.0, channel_count=w.x_channel_count,
                       channel_mult=w.x_channel_mult)


def make_bias(w: Workload):
    if w.bias_sigma is None:
        return None
    return draw_bias(w.seed, w.N, sigma=w.bias_sigma)


def algorithmic_bytes(w: Workload, M: int, N: int | None = None, K: int | None = None) -> int:
    """Bytes the linear must move once: packed W + scales + aux + X + Y + bias."""
    N = w.N if N is None else N
    K = w.K if K is None else K
    return packed_bytes(w.fmt, N, K, w.group_size) + 2 * M * K + 2 * M * N + \
        (2 * N if w.bias_sigma is not None else 0)


def packed_bytes(fmt: str, N: int, K: int, G: int) -> int:
    """Weight-side bytes: codes + scales + auxiliary data, for the given format."""
    if fmt == "int4_sym":
        return N * K // 2 + 2 * N * (K // G)
    if fmt == "int2_sym":
        return N * K // 4 + 2 * N * (K // G)
    if fmt == "int3_sym":
        return N * K * 3 // 8 + 2 * N * (K // G)
    if fmt == "int4_asym":
        return N * K // 2 + 2 * N * (K // G) + N * (K // G) // 2
    if fmt == "int8_sym":
        return N * K + 2 * N * (K // G)
    if fmt == "cb4":
        return N * K // 2 + 2 * N + 64
    if fmt == "nvfp4":
        return N * K // 2 + N * (K // 16) + 4
    if fmt == "mxfp4":
        return N * K // 2 + N * (K // 32)
    if fmt in ("fp8_e4m3", "fp8_e5m2"):
        return N * K + 4 * N * (K // G)
    raise ValueError(fmt)


def flops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K


@dataclass(frozen=True)
class MoEWorkload:
    """A mixture-of-experts layer: E experts of one format, each [N, K];
    `tokens` tokens routed to `topk` experts each, so tokens * topk rows of x
    sorted by expert, with skewed (Zipf-like) per-expert counts."""
    name: str
    fmt: str
    E: int
    N: int
    K: int
    tokens: int
    topk: int
    group_size: int
    seed: int
    note: str = ""

    @property
    def rows(self) -> int:
        return self.tokens * self.topk


MOE_DECODE = MoEWorkload("moe_int4_decode", "int4_sym", E=64, N=2048, K=2048, tokens=64, topk=8,
                         group_size=128, seed=7,
                         note="decode-like routing: 64 tokens x top-8 over 64 INT4 experts")
MOE_PREFILL = MoEWorkload("moe_int4_prefill", "int4_sym", E=64, N=2048, K=2048, tokens=4096,
                          topk=8, group_size=128, seed=8,
                          note="prefill-like routing: 4096 tokens x top-8 over 64 INT4 experts")
MOE = {w.name: w for w in (MOE_DECODE, MOE_PREFILL)}


def moe_counts(w: MoEWorkload) -> np.ndarray:
    """Rows per expert (sum = tokens * topk): a multinomial draw with Zipf(1.1)
    expert weights in a seeded random order."""
    rng = np.random.default_rng(w.seed)
    p = 1.0 / np.arange(1, w.E + 1) ** 1.1
    p = p[rng.permutation(w.E)]
    return rng.multinomial(w.rows, p / p.sum()).astype(np.int64)


def moe_weight(w: MoEWorkload, e: int) -> np.ndarray:
    """Expert e's dense fp32 weight [N, K] ~ N(0, 0.02^2)."""
    return weight(w.seed * 1000 + e, w.N, w.K, sigma=0.02)


def moe_x(w: MoEWorkload) -> np.ndarray:
    return activations(w.seed, w.rows, w.K)


def moe_bytes(w: MoEWorkload, counts) -> int:
    """Algorithmic bytes: the packed weights of every expert with rows, X, Y."""
    used = int(np.count_nonzero(np.asarray(counts)))
    return used * packed_bytes(w.fmt, w.N, w.K, w.group_size) + 2 * w.rows * (w.K + w.N)
