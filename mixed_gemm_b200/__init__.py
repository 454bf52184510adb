"""Python binding of the C-ABI library ``libwq.so`` (declared in include/wq.h).

Argument marshalling only: every step of the quantized linear runs in the
library's CUDA kernels.  Functions carry the C names (``wq_linear``,
``wq_pack`` ...) and accept torch tensors (device memory; the pointer is
``data_ptr()``) or raw integer addresses, plus an optional stream (a
``torch.cuda.Stream``, a raw ``cudaStream_t`` integer, or None for torch's
current stream).  A non-zero status raises ``WQError``.

There is no fallback: if ``libwq.so`` is missing or cannot be loaded, the
import fails.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwq.so")

FORMATS = {"int4_sym": 0, "int4_asym": 1, "int8_sym": 2, "cb4": 3, "nvfp4": 4, "mxfp4": 5,
           "fp8_e4m3": 6, "fp8_e5m2": 7, "int2_sym": 8, "int3_sym": 9}
FORMAT_NAMES = {v: k for k, v in FORMATS.items()}

WQ_OK = 0
WQ_ERR_INVALID_ARG = 1
WQ_ERR_UNSUPPORTED = 2
WQ_ERR_ALIGNMENT = 3
WQ_ERR_CUDA = 4
WQ_ERR_DEVICE_CHECK = 5


class WQError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {wq_status_string(status)} (status {status})")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with mixed_gemm_b200._build.build() "
                      "(nvcc, sm_100a); there is no non-CUDA implementation")
_lib = ctypes.CDLL(LIB_PATH)

_i64, _int, _ptr, _sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.POINTER(ctypes.c_size_t)
_SIGS = {
    "wq_status_string": ([_int], ctypes.c_char_p),
    "wq_canonical_sizes": ([_int, _i64, _i64, _int, _sz, _sz, _sz], _int),
    "wq_packed_sizes": ([_int, _i64, _i64, _int, _sz, _sz, _sz], _int),
    "wq_pack": ([_int, _i64, _i64, _int, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr], _int),
    "wq_unpack": ([_int, _i64, _i64, _int, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr], _int),
    "wq_dequant": ([_int, _i64, _i64, _int, _ptr, _ptr, _ptr, _ptr, _ptr], _int),
    "wq_linear": ([_ptr, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _int, _int, _ptr, _ptr], _int),
    "wq_linear_grouped_dev": ([_ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _i64, _int,
                               _int, _ptr, _ptr], _int),
    "wq_linear_swiglu": ([_ptr, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _int, _int, _ptr,
                          ctypes.c_size_t, _ptr, _ptr], _int),
    "wq_linear_grouped": ([_ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _int, _int,
                           _ptr, _ptr], _int),
    "wq_addmm_requant": ([_int, _i64, _i64, _int, _ptr, _ptr, _ptr, _ptr, _i64, ctypes.c_double,
                          ctypes.c_double, _int, ctypes.c_uint64, _ptr], _int),
    "wq_linear_swiglu_static": ([_ptr, _ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _int, _int, _ptr,
                                 _ptr], _int),
    "wq_quantize": ([_int, _i64, _i64, _int, _ptr, _ptr, _ptr, _ptr, _ptr], _int),
    "wq_linear_a8_workspace_size": ([_i64, _i64, _sz], _int),
    "wq_linear_a8": ([_ptr, _ptr, _ptr, _ptr, _i64, _i64, _i64, _int, _int, _ptr, ctypes.c_size_t,
                      _ptr, _ptr], _int),
    "wq_quantize_act_int8": ([_ptr, _i64, _i64, _ptr, _ptr, _ptr], _int),
    "wq_lloyd_max_centroids": ([_int, ctypes.POINTER(ctypes.c_float)], _int),
    "wq_device_sm_count": ([ctypes.POINTER(ctypes.c_int)], _int),
    "wq_device_error": ([ctypes.POINTER(ctypes.c_uint), _int], _int),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def _addr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _fmt(f):
    return FORMATS[f] if isinstance(f, str) else int(f)


def _check(st: int, where: str):
    if st != WQ_OK:
        raise WQError(st, where)


def wq_status_string(status: int) -> str:
    return _lib.wq_status_string(status).decode()


def wq_canonical_sizes(fmt, N: int, K: int, group_size: int = 0):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.wq_canonical_sizes(_fmt(fmt), N, K, group_size, ctypes.byref(a), ctypes.byref(b),
                                   ctypes.byref(c)), "wq_canonical_sizes")
    return a.value, b.value, c.value


def wq_packed_sizes(fmt, N: int, K: int, group_size: int = 0):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.wq_packed_sizes(_fmt(fmt), N, K, group_size, ctypes.byref(a), ctypes.byref(b),
                                ctypes.byref(c)), "wq_packed_sizes")
    return a.value, b.value, c.value


def wq_pack(fmt, N, K, group_size, codes, scales, aux, packed_w, packed_scales, packed_aux,
            stream=None):
    _check(_lib.wq_pack(_fmt(fmt), N, K, group_size, _addr(codes), _addr(scales), _addr(aux),
                        _addr(packed_w), _addr(packed_scales), _addr(packed_aux), _stream(stream)),
           "wq_pack")


def wq_unpack(fmt, N, K, group_size, packed_w, packed_scales, packed_aux, codes, scales, aux,
              stream=None):
    _check(_lib.wq_unpack(_fmt(fmt), N, K, group_size, _addr(packed_w), _addr(packed_scales),
                          _addr(packed_aux), _addr(codes), _addr(scales), _addr(aux),
                          _stream(stream)), "wq_unpack")


def wq_dequant(fmt, N, K, group_size, packed_w, packed_scales, packed_aux, out_f32, stream=None):
    _check(_lib.wq_dequant(_fmt(fmt), N, K, group_size, _addr(packed_w), _addr(packed_scales),
                           _addr(packed_aux), _addr(out_f32), _stream(stream)), "wq_dequant")


def wq_linear(x, packed_w, scales, aux, bias, M, N, K, fmt, group_size, out, stream=None):
    _check(_lib.wq_linear(_addr(x), _addr(packed_w), _addr(scales), _addr(aux), _addr(bias), M, N,
                          K, _fmt(fmt), group_size, _addr(out), _stream(stream)), "wq_linear")


def wq_linear_swiglu(x2, packed_w, scales, aux, bias, M, N, K, fmt, group_size, workspace,
                     workspace_bytes, out, stream=None):
    _check(_lib.wq_linear_swiglu(_addr(x2), _addr(packed_w), _addr(scales), _addr(aux),
                                 _addr(bias), M, N, K, _fmt(fmt), group_size, _addr(workspace),
                                 int(workspace_bytes), _addr(out), _stream(stream)),
           "wq_linear_swiglu")


def wq_linear_grouped(x, packed_w, scales, aux, bias, offsets, N, K, fmt, group_size, out,
                      stream=None):
    """``packed_w``, ``scales``, ``aux``, ``bias``: sequences of E device
    tensors / addresses (``aux`` and ``bias`` may be None); ``offsets``: E + 1
    row offsets (host integers)."""
    E = len(packed_w)
    arr = ctypes.c_void_p * E

    def ptrs(seq):
        if seq is None:
            return None
        return arr(*[_addr(t) for t in seq])

    offs = (ctypes.c_int64 * (E + 1))(*[int(o) for o in offsets])
    _check(_lib.wq_linear_grouped(_addr(x), ptrs(packed_w), ptrs(scales), ptrs(aux), ptrs(bias),
                                  offs, E, N, K, _fmt(fmt), group_size, _addr(out),
                                  _stream(stream)), "wq_linear_grouped")


def wq_linear_grouped_dev(x, packed_w, scales, aux, bias, offsets, E, T, N, K, fmt, group_size,
                          out, stream=None):
    """One launch over E stacked experts; ``offsets``: device int64 [E + 1]."""
    _check(_lib.wq_linear_grouped_dev(_addr(x), _addr(packed_w), _addr(scales), _addr(aux),
                                      _addr(bias), _addr(offsets), E, T, N, K, _fmt(fmt),
                                      group_size, _addr(out), _stream(stream)),
           "wq_linear_grouped_dev")


def wq_addmm_requant(fmt, N, K, group_size, packed_w, packed_scales, mat1, mat2, rank, alpha,
                     beta=1.0, seed=None, stream=None):
    _check(_lib.wq_addmm_requant(_fmt(fmt), N, K, group_size, _addr(packed_w),
                                 _addr(packed_scales), _addr(mat1), _addr(mat2), rank,
                                 float(alpha), float(beta), 0 if seed is None else 1,
                                 0 if seed is None else int(seed), _stream(stream)),
           "wq_addmm_requant")


def wq_linear_swiglu_static(x2, packed_w, scales, aux, bias, M, N, K, fmt, group_size, out,
                            stream=None):
    _check(_lib.wq_linear_swiglu_static(_addr(x2), _addr(packed_w), _addr(scales), _addr(aux),
                                        _addr(bias), M, N, K, _fmt(fmt), group_size, _addr(out),
                                        _stream(stream)), "wq_linear_swiglu_static")


def wq_quantize(fmt, N, K, group_size, w_f32, codes, scales, aux, stream=None):
    _check(_lib.wq_quantize(_fmt(fmt), N, K, group_size, _addr(w_f32), _addr(codes),
                            _addr(scales), _addr(aux), _stream(stream)), "wq_quantize")


def wq_linear_a8_workspace_size(M: int, K: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib.wq_linear_a8_workspace_size(M, K, ctypes.byref(n)), "wq_linear_a8_workspace_size")
    return n.value


def wq_linear_a8(x, packed_w, scales, bias, M, N, K, fmt, group_size, workspace, workspace_bytes,
                 out, stream=None):
    _check(_lib.wq_linear_a8(_addr(x), _addr(packed_w), _addr(scales), _addr(bias), M, N, K,
                             _fmt(fmt), group_size, _addr(workspace), int(workspace_bytes),
                             _addr(out), _stream(stream)), "wq_linear_a8")


def wq_quantize_act_int8(x, M, K, xq, sx, stream=None):
    _check(_lib.wq_quantize_act_int8(_addr(x), M, K, _addr(xq), _addr(sx), _stream(stream)),
           "wq_quantize_act_int8")


def wq_lloyd_max_centroids(bits: int = 4):
    import numpy as np
    out = np.zeros((1 << bits,), dtype=np.float32)
    _check(_lib.wq_lloyd_max_centroids(bits, out.ctypes.data_as(ctypes.POINTER(ctypes.c_float))),
           "wq_lloyd_max_centroids")
    return out


def wq_device_error(clear: bool = True) -> int:
    """The kernels' error word (0 when every bounded wait completed)."""
    v = ctypes.c_uint(0)
    st = _lib.wq_device_error(ctypes.byref(v), 1 if clear else 0)
    if st not in (WQ_OK, WQ_ERR_DEVICE_CHECK):
        raise WQError(st, "wq_device_error")
    return v.value


def wq_device_sm_count() -> int:
    n = ctypes.c_int(0)
    _check(_lib.wq_device_sm_count(ctypes.byref(n)), "wq_device_sm_count")
    return n.value


from .api import (PackedWeight, linear, linear_a8, linear_grouped, linear_moe,  # noqa: E402,F401
                  linear_swiglu, pack, quantize_and_pack, stack_experts)
