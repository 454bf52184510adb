"""The kernels' bounded waits, made to run out on purpose in a test build.

A second copy of the library is compiled with -DWQ_FAULT_TEST (short wait
limits; environment switches that drop exactly one mbarrier arrival: the
first dequant warp's arrival on one A-tile barrier of the tcgen05 kernel, or
block 0's arrival on the decode kernel's activation-slice barrier, with its
copies).  No copy is altered and nothing faults: the waiting thread gives up,
records its bit in the kernel's error word and the thread block winds down.
The tests check that the call returns, the word reports the bit, and a
normal call on the same CUDA context afterwards matches the oracle.  The
regular library never contains these switches."""
from __future__ import annotations

import ctypes
import os

import numpy as np
import pytest
import torch

import synth
from gpu_cases import bf16_bits, check_close, dev_bf16, pack_on_gpu, small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faultlib(tmp_path_factory):
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location(
        "_wq_build_fault", os.path.join(root, "mixed_gemm_b200", "_build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    d = tmp_path_factory.mktemp("wq_fault")
    path = b.build(force=True, extra=["-DWQ_FAULT_TEST"], out_path=str(d / "libwq_fault.so"),
                   obj_dir=str(d / "obj"))
    lib = ctypes.CDLL(path)
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.wq_linear.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, vp]
    lib.wq_linear.restype = i32
    lib.wq_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), i32]
    lib.wq_device_error.restype = i32
    return lib


def _err(lib) -> int:
    v = ctypes.c_uint(0)
    lib.wq_device_error(ctypes.byref(v), 1)
    return v.value


def _call(lib, wq, pw, x, y, M):
    s = torch.cuda.current_stream().cuda_stream
    st = lib.wq_linear(x.data_ptr(), pw.w.data_ptr(), pw.scales.data_ptr(), None, None, M, pw.N,
                       pw.K, wq.FORMATS[pw.fmt], pw.group_size, y.data_ptr(), s)
    torch.cuda.synchronize()
    return st


@pytest.mark.parametrize("which", ["prefill", "decode"])
def test_wait_runs_out_and_context_stays_usable(wq, orc, faultlib, which):
    fmt, G, N, K = "int4_sym", 64, 1024, 512
    M = 300 if which == "prefill" else 4
    W, (codes, scales, aux) = small_case(orc, fmt, N, K, G, seed=91)
    pw = pack_on_gpu(wq, fmt, N, K, G, codes, scales, aux)
    xh = synth.activations(92, M, K)
    x = dev_bf16(xh)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    _err(faultlib)
    var = "WQ_FAULT_PREFILL_STAGE" if which == "prefill" else "WQ_FAULT_DECODE_SKIP_X"
    os.environ[var] = "2" if which == "prefill" else "1"
    try:
        st = _call(faultlib, wq, pw, x, y, M)
    finally:
        os.environ.pop(var, None)
    assert st == 0                                           # the launch itself succeeded
    err = _err(faultlib)
    bit = 8 if which == "prefill" else 128                   # MMA wait / activation-slice wait
    assert err & bit, f"error word {err:#x}"
    assert _err(faultlib) == 0                               # read and cleared
    # the same context: the test build without the switch, then the regular library
    ref, _ = orc.linear(xh, orc.dequant(fmt, codes, scales, aux, N, K, G), None)
    y.fill_(float("nan"))
    assert _call(faultlib, wq, pw, x, y, M) == 0 and _err(faultlib) == 0
    check_close(bf16_bits(y), ref, f"{which}: test build after the timed-out call")
    y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    wq.wq_linear(x, pw.w, pw.scales, None, None, M, N, K, fmt, G, y2)
    torch.cuda.synchronize()
    assert wq.wq_device_error() == 0
    check_close(bf16_bits(y2), ref, f"{which}: regular library after the timed-out call")
