"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module draws inputs only: the dense fp32 weight matrix that the offline
quantizers consume, the bf16 activations and the bf16 bias.  It holds none of
the method's arithmetic.  The drawing itself lives in ``synth.c`` (SplitMix64
streams, Box-Muller normals, Student-t from normals); this file builds it with
gcc, loads it with ctypes and returns numpy arrays.

Workload recipes (shapes, seeds, distributions) are in ``synth.workloads``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` beside it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        i64, u64, dbl, ptr = ctypes.c_int64, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
        lib.synth_weight_f32.argtypes = [u64, i64, i64, ctypes.c_int, dbl, i64, dbl, ptr]
        lib.synth_act_bf16.argtypes = [u64, i64, i64, dbl, i64, dbl, ptr]
        lib.synth_bias_bf16.argtypes = [u64, i64, dbl, ptr]
        lib.synth_distinct_positions.argtypes = [u64, u64, i64, i64, ptr]
        lib.synth_uniform_f64.argtypes = [u64, u64, i64, i64, ptr]
        lib.synth_normal_f64.argtypes = [u64, u64, i64, i64, ptr]
        lib.synth_student5_f64.argtypes = [u64, u64, i64, i64, ptr]
        lib.synth_splitmix64.argtypes = [u64, u64]
        lib.synth_splitmix64.restype = u64
        lib.synth_f64_to_bf16.argtypes = [ptr, i64, ptr]
        for name in ("synth_weight_f32", "synth_act_bf16", "synth_bias_bf16",
                     "synth_distinct_positions", "synth_uniform_f64", "synth_normal_f64",
                     "synth_student5_f64", "synth_f64_to_bf16"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


# ---------------------------------------------------------------- tensors
def weight(seed: int, N: int, K: int, dist: str = "normal", sigma: float = 0.02,
           outlier_count: int = 0, outlier_mult: float = 1.0) -> np.ndarray:
    """Dense W[N, K] fp32: ``sigma * N(0,1)`` or ``sigma * t(5)``, optional outliers."""
    lib = _load()
    out = np.empty((N, K), dtype=np.float32)
    d = {"normal": 0, "student5": 1}[dist]
    _check(lib.synth_weight_f32(seed, N, K, d, sigma, outlier_count, outlier_mult, _ptr(out)),
           "synth_weight_f32")
    return out


def activations(seed: int, M: int, K: int, sigma: float = 1.0, channel_count: int = 0,
                channel_mult: float = 1.0) -> np.ndarray:
    """X[M, K] as bf16 bit patterns (uint16): ``sigma * N(0,1)``, optional hot channels."""
    lib = _load()
    out = np.empty((M, K), dtype=np.uint16)
    _check(lib.synth_act_bf16(seed, M, K, sigma, channel_count, channel_mult, _ptr(out)),
           "synth_act_bf16")
    return out


def bias(seed: int, N: int, sigma: float = 0.01) -> np.ndarray:
    """bias[N] as bf16 bit patterns (uint16): ``sigma * N(0,1)``."""
    lib = _load()
    out = np.empty((N,), dtype=np.uint16)
    _check(lib.synth_bias_bf16(seed, N, sigma, _ptr(out)), "synth_bias_bf16")
    return out


def distinct_positions(seed: int, tensor_id: int, range_: int, count: int) -> np.ndarray:
    lib = _load()
    out = np.empty((count,), dtype=np.int64)
    _check(lib.synth_distinct_positions(seed, tensor_id, range_, count, _ptr(out)),
           "synth_distinct_positions")
    return out


def uniform_stream(seed: int, tensor_id: int, start: int, n: int) -> np.ndarray:
    lib = _load()
    out = np.empty((n,), dtype=np.float64)
    _check(lib.synth_uniform_f64(seed, tensor_id, start, n, _ptr(out)), "synth_uniform_f64")
    return out


def normal_stream(seed: int, tensor_id: int, start: int, n: int) -> np.ndarray:
    lib = _load()
    out = np.empty((n,), dtype=np.float64)
    _check(lib.synth_normal_f64(seed, tensor_id, start, n, _ptr(out)), "synth_normal_f64")
    return out


def student5_stream(seed: int, tensor_id: int, start: int, n: int) -> np.ndarray:
    lib = _load()
    out = np.empty((n,), dtype=np.float64)
    _check(lib.synth_student5_f64(seed, tensor_id, start, n, _ptr(out)), "synth_student5_f64")
    return out


def splitmix64(key: int, i: int) -> int:
    return int(_load().synth_splitmix64(key, i))


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    lib = _load()
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    _check(lib.synth_f64_to_bf16(_ptr(a), a.size, _ptr(out)), "synth_f64_to_bf16")
    return out
