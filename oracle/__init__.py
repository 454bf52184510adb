"""ORACLE - test infrastructure, not part of the library.

Plain CPU statement of the weight-only quantized linear (``oracle.c``), loaded
with ctypes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package; the library never does.

Functions take and return numpy arrays in the canonical (pre-pack) layouts
listed in ``oracle.c``.  bf16 tensors travel as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FORMATS = {"int4_sym": 0, "int4_asym": 1, "int8_sym": 2, "cb4": 3, "nvfp4": 4, "mxfp4": 5,
           "fp8_e4m3": 6, "fp8_e5m2": 7, "int2_sym": 8, "int3_sym": 9}


def build(force: bool = False, extra_flags=(), out_path: str | None = None,
          src: str | None = None) -> str:
    """Compile ``oracle.c`` with gcc.  ``src``/``out_path`` let a test build a
    deliberately altered copy of the source elsewhere."""
    out = out_path or _LIB_PATH
    src = src or _SRC
    if (not force and out_path is None and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", *extra_flags, "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _declare(lib):
    i64, ptr, c_int, dbl = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_double
    sig = {
        "orc_bf16_to_f32": ([ctypes.c_uint16], ctypes.c_float),
        "orc_f64_to_bf16": ([dbl], ctypes.c_uint16),
        "orc_e2m1_value": ([c_int], dbl),
        "orc_e2m1_encode": ([dbl], c_int),
        "orc_e4m3_value": ([c_int], dbl),
        "orc_e4m3_encode": ([dbl], c_int),
        "orc_e5m2_value": ([c_int], dbl),
        "orc_e5m2_encode": ([dbl], c_int),
        "orc_quant_int_sym": ([ptr, i64, i64, c_int, c_int, ptr, ptr], c_int),
        "orc_quant_int4_asym": ([ptr, i64, i64, c_int, ptr, ptr, ptr], c_int),
        "orc_lloyd_max_gaussian": ([c_int, ptr, ptr, ptr, ptr], c_int),
        "orc_quant_cb4": ([ptr, i64, i64, ptr, ptr, ptr], c_int),
        "orc_quant_nvfp4": ([ptr, i64, i64, ptr, ptr, ptr], c_int),
        "orc_quant_mxfp4": ([ptr, i64, i64, ptr, ptr], c_int),
        "orc_quant_fp8_e4m3": ([ptr, i64, i64, c_int, ptr, ptr], c_int),
        "orc_quant_fp8_e5m2": ([ptr, i64, i64, c_int, ptr, ptr], c_int),
        "orc_e8m0_value": ([c_int], dbl),
        "orc_dequant": ([c_int, i64, i64, c_int, ptr, ptr, ptr, ptr], c_int),
        "orc_linear": ([ptr, ptr, ptr, i64, i64, i64, ptr, ptr], c_int),
        "orc_linear_sampled": ([c_int, i64, i64, c_int, ptr, ptr, ptr, ptr, ptr, i64, ptr, ptr,
                                ptr, ptr], c_int),
        "orc_threads": ([], c_int),
        "orc_set_threads": ([c_int], None),
        "orc_silu": ([dbl], dbl),
        "orc_swiglu": ([ptr, i64, i64, ptr], c_int),
        "orc_quant_act_int8": ([ptr, i64, i64, ptr, ptr], c_int),
        "orc_linear_a8": ([c_int, ptr, ptr, i64, i64, c_int, ptr, ptr, ptr, i64, ptr, ptr], c_int),
        "orc_round_bf16_array": ([ptr, i64, ptr], c_int),
        "orc_addmm_requant_int8": ([ptr, ptr, i64, i64, c_int, ptr, ptr, i64, dbl, dbl, c_int,
                                    ctypes.c_uint64], c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res


def load(path: str | None = None):
    """The oracle library (built on first use).  ``path`` loads another build."""
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
        _declare(lib)
        return lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            _declare(lib)
            _lib = lib
        return _lib


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "contiguous numpy array expected"
    return a.ctypes.data


def _ok(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


class Oracle:
    """Thin numpy front end over one build of ``oracle.c``."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    # ---- scalar codecs
    def bf16_to_f32(self, bits: int) -> float:
        return float(self.lib.orc_bf16_to_f32(bits))

    def f64_to_bf16(self, v: float) -> int:
        return int(self.lib.orc_f64_to_bf16(v))

    def e2m1_value(self, code: int) -> float:
        return float(self.lib.orc_e2m1_value(code))

    def e2m1_encode(self, r: float) -> int:
        return int(self.lib.orc_e2m1_encode(r))

    def e4m3_value(self, code: int) -> float:
        return float(self.lib.orc_e4m3_value(code))

    def e4m3_encode(self, d: float) -> int:
        return int(self.lib.orc_e4m3_encode(d))

    def e5m2_value(self, code: int) -> float:
        return float(self.lib.orc_e5m2_value(code))

    def e5m2_encode(self, d: float) -> int:
        return int(self.lib.orc_e5m2_encode(d))

    def e8m0_value(self, code: int) -> float:
        return float(self.lib.orc_e8m0_value(code))

    # ---- quantizers -> canonical layout
    def quantize(self, fmt: str, W: np.ndarray, group_size: int = 0, centroids=None):
        """Returns (codes, scales, aux) in the canonical layout of ``fmt``."""
        W = np.ascontiguousarray(W, dtype=np.float32)
        N, K = W.shape
        G = group_size
        if fmt in ("int2_sym", "int3_sym", "int4_sym", "int8_sym"):
            bits = {"int2_sym": 2, "int3_sym": 3, "int4_sym": 4, "int8_sym": 8}[fmt]
            codes = np.zeros((N, K * bits // 8), dtype=np.int8 if bits == 8 else np.uint8)
            scales = np.zeros((N, K // G), dtype=np.uint16)
            _ok(self.lib.orc_quant_int_sym(_p(W), N, K, G, bits, _p(codes), _p(scales)), fmt)
            return codes, scales, None
        if fmt == "int4_asym":
            codes = np.zeros((N, K // 2), dtype=np.uint8)
            scales = np.zeros((N, K // G), dtype=np.uint16)
            zeros = np.zeros((N, K // G), dtype=np.uint8)
            _ok(self.lib.orc_quant_int4_asym(_p(W), N, K, G, _p(codes), _p(scales), _p(zeros)), fmt)
            return codes, scales, zeros
        if fmt == "cb4":
            c = self.lloyd_max(16)[1] if centroids is None else np.ascontiguousarray(
                centroids, dtype=np.float32)
            codes = np.zeros((N, K // 2), dtype=np.uint8)
            norms = np.zeros((N,), dtype=np.uint16)
            _ok(self.lib.orc_quant_cb4(_p(W), N, K, _p(c), _p(codes), _p(norms)), fmt)
            return codes, norms, c
        if fmt == "nvfp4":
            codes = np.zeros((N, K // 2), dtype=np.uint8)
            bs = np.zeros((N, K // 16), dtype=np.uint8)
            ts = np.zeros((1,), dtype=np.float32)
            _ok(self.lib.orc_quant_nvfp4(_p(W), N, K, _p(codes), _p(bs), _p(ts)), fmt)
            return codes, bs, ts
        if fmt == "mxfp4":
            codes = np.zeros((N, K // 2), dtype=np.uint8)
            bs = np.zeros((N, K // 32), dtype=np.uint8)
            _ok(self.lib.orc_quant_mxfp4(_p(W), N, K, _p(codes), _p(bs)), fmt)
            return codes, bs, None
        if fmt in ("fp8_e4m3", "fp8_e5m2"):
            codes = np.zeros((N, K), dtype=np.uint8)
            scales = np.zeros((N, K // G), dtype=np.float32)
            fn = self.lib.orc_quant_fp8_e4m3 if fmt == "fp8_e4m3" else self.lib.orc_quant_fp8_e5m2
            _ok(fn(_p(W), N, K, G, _p(codes), _p(scales)), fmt)
            return codes, scales, None
        raise ValueError(fmt)

    def lloyd_max(self, levels: int = 16):
        """(c64, c32, iterations, mse) of the Lloyd-Max quantizer of N(0,1)."""
        c64 = np.zeros((levels,), dtype=np.float64)
        c32 = np.zeros((levels,), dtype=np.float32)
        it = ctypes.c_int(0)
        mse = ctypes.c_double(0.0)
        _ok(self.lib.orc_lloyd_max_gaussian(levels, _p(c64), _p(c32), ctypes.byref(it),
                                            ctypes.byref(mse)), "lloyd_max")
        return c64, c32, it.value, mse.value

    # ---- dequant / linear
    def dequant(self, fmt: str, codes, scales, aux, N: int, K: int, group_size: int = 0):
        out = np.zeros((N, K), dtype=np.float32)
        _ok(self.lib.orc_dequant(FORMATS[fmt], N, K, group_size, _p(codes), _p(scales), _p(aux),
                                 _p(out)), "dequant")
        return out

    def linear(self, x_bits: np.ndarray, dq: np.ndarray, bias_bits=None):
        """(y_bf16_bits [M,N], y_f64 [M,N]) for y = x . dq^T + bias."""
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        dq = np.ascontiguousarray(dq, dtype=np.float32)
        M, K = x_bits.shape
        N = dq.shape[0]
        assert dq.shape[1] == K
        y = np.zeros((M, N), dtype=np.uint16)
        y64 = np.zeros((M, N), dtype=np.float64)
        b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
        _ok(self.lib.orc_linear(_p(x_bits), _p(dq), _p(b), M, N, K, _p(y), _p(y64)), "linear")
        return y, y64

    def linear_full(self, x_bits: np.ndarray, dq: np.ndarray, bias_bits=None,
                    rows_per_chunk: int = 4096):
        """(y_bf16_bits [M,N], y_f64 [M,N]) for y = x . dq^T + bias, with the
        fp64 product taken by numpy's fp64 matmul (a library primitive)
        instead of orc_linear's loop, so that full-size outputs cost seconds.

        Same definition as ``linear``: exact bf16 and fp32 operands widened
        to fp64, one fp64 sum per output plus the bias, rounded once to bf16
        by ``orc_round_bf16_array``.  Only the order of the fp64 additions
        differs (fp64 error far below half a bf16 step), which the pins
        check against ``linear``."""
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        M, K = x_bits.shape
        N = dq.shape[0]
        assert dq.shape[1] == K
        xf = bits_to_f32(x_bits).astype(np.float64)
        y64 = np.empty((M, N), dtype=np.float64)
        for n0 in range(0, N, rows_per_chunk):
            n1 = min(N, n0 + rows_per_chunk)
            y64[:, n0:n1] = xf @ np.asarray(dq[n0:n1], dtype=np.float32).astype(np.float64).T
        if bias_bits is not None:
            y64 += bits_to_f32(np.asarray(bias_bits, dtype=np.uint16)).astype(np.float64)[None, :]
        y = np.zeros((M, N), dtype=np.uint16)
        _ok(self.lib.orc_round_bf16_array(_p(y64), M * N, _p(y)), "round_bf16_array")
        return y, y64

    def quant_act_int8(self, x_bits: np.ndarray):
        """Per-token INT8 activation quantization: (x_q int8 [M, K], s_x f32 [M])."""
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        M, K = x_bits.shape
        xq = np.zeros((M, K), dtype=np.int8)
        sx = np.zeros((M,), dtype=np.float32)
        _ok(self.lib.orc_quant_act_int8(_p(x_bits), M, K, _p(xq), _p(sx)), "quant_act_int8")
        return xq, sx

    def linear_a8(self, fmt: str, codes, scales, N: int, K: int, G: int, x_bits, bias_bits=None):
        """(y bf16 bits, y fp64) of the activation-quantized linear (INT4 / INT8 sym)."""
        xq, sx = self.quant_act_int8(x_bits)
        M = xq.shape[0]
        y = np.zeros((M, N), dtype=np.uint16)
        y64 = np.zeros((M, N), dtype=np.float64)
        b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
        _ok(self.lib.orc_linear_a8(FORMATS[fmt], _p(np.ascontiguousarray(codes)),
                                   _p(np.ascontiguousarray(scales, dtype=np.uint16)), N, K, G,
                                   _p(xq), _p(sx), _p(b), M, _p(y), _p(y64)), "linear_a8")
        return y, y64

    def linear_a8_full(self, codes, scales, N: int, K: int, G: int, x_bits, bias_bits=None):
        """(y bf16 bits, y fp64) of the activation-quantized linear for INT8
        or INT4 sym weights, with each group's integer sum taken by numpy's fp64
        matmul (exact: every partial sum is an integer below 2^53) instead
        of orc_linear_a8's loop, so that full sizes cost seconds.  The codes
        come from orc_quant_act_int8 and the fp64 accumulation over groups
        follows orc_linear_a8 step for step ((s_w * s_x) * isum, increasing g,
        then the bias), so the fp64 result is the same number."""
        xq, sx = self.quant_act_int8(x_bits)
        M = xq.shape[0]
        if np.asarray(codes).size * 2 == N * K:      # INT4 sym: two's complement nibbles
            c = np.ascontiguousarray(codes, dtype=np.uint8).reshape(N, K // 2)
            nib = np.empty((N, K), dtype=np.int16)
            nib[:, 0::2] = c & 15
            nib[:, 1::2] = c >> 4
            wq = (nib - 16 * (nib > 7)).astype(np.int8)
        else:
            wq = np.ascontiguousarray(codes, dtype=np.int8).reshape(N, K)
        sw = bits_to_f32(np.ascontiguousarray(scales, dtype=np.uint16).reshape(N, K // G))
        sw = sw.astype(np.float64)
        sxd = sx.astype(np.float64)
        y64 = np.zeros((M, N), dtype=np.float64)
        for g in range(K // G):
            isum = xq[:, g * G:(g + 1) * G].astype(np.float64) @ \
                wq[:, g * G:(g + 1) * G].astype(np.float64).T
            y64 += (sw[None, :, g] * sxd[:, None]) * isum
        if bias_bits is not None:
            y64 = y64 + bits_to_f32(np.asarray(bias_bits, dtype=np.uint16)).astype(np.float64)[None, :]
        y = np.zeros((M, N), dtype=np.uint16)
        _ok(self.lib.orc_round_bf16_array(_p(y64), M * N, _p(y)), "round_bf16_array")
        return y, y64

    def silu(self, g: float) -> float:
        return float(self.lib.orc_silu(g))

    def swiglu(self, x2_bits: np.ndarray) -> np.ndarray:
        """bf16 bits [M, K] of up * silu(gate) for an input [M, 2K] = [up | gate]."""
        x2_bits = np.ascontiguousarray(x2_bits, dtype=np.uint16)
        M, K2 = x2_bits.shape
        assert K2 % 2 == 0
        a = np.zeros((M, K2 // 2), dtype=np.uint16)
        _ok(self.lib.orc_swiglu(_p(x2_bits), M, K2 // 2, _p(a)), "swiglu")
        return a

    def addmm_requant_int8(self, codes, scales, G: int, mat1_bits, mat2_bits, alpha: float,
                           beta: float, seed=None):
        """New canonical INT8 codes after weight = beta * weight + alpha * mat1 @ mat2,
        requantized with the unchanged scales (nearest, or stochastic with a seed)."""
        out = np.ascontiguousarray(codes, dtype=np.int8).copy()
        N, K = out.shape
        m1 = np.ascontiguousarray(mat1_bits, dtype=np.uint16)
        m2 = np.ascontiguousarray(mat2_bits, dtype=np.uint16)
        R = m1.shape[1]
        sc = np.ascontiguousarray(scales, dtype=np.uint16)
        _ok(self.lib.orc_addmm_requant_int8(_p(out), _p(sc), N, K, G, _p(m1), _p(m2), R,
                                            float(alpha), float(beta), 0 if seed is None else 1,
                                            0 if seed is None else int(seed)), "addmm_requant")
        return out

    def linear_sampled(self, fmt: str, codes, scales, aux, N: int, K: int, group_size: int,
                       x_bits, bias_bits, ms, ns):
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        ns = np.ascontiguousarray(ns, dtype=np.int64)
        S = ms.size
        y = np.zeros((S,), dtype=np.uint16)
        y64 = np.zeros((S,), dtype=np.float64)
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
        _ok(self.lib.orc_linear_sampled(FORMATS[fmt], N, K, group_size, _p(codes), _p(scales),
                                        _p(aux), _p(x_bits), _p(b), S, _p(ms), _p(ns), _p(y),
                                        _p(y64)), "linear_sampled")
        return y, y64

    def set_threads(self, n: int) -> None:
        self.lib.orc_set_threads(int(n))

    def threads(self) -> int:
        return int(self.lib.orc_threads())


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
