"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, sizes buffers, and rejects bad arguments before launching anything."""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wq.h")

import mixed_gemm_b200 as wqm  # noqa: E402


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported():
    names = _declared()
    assert "wq_linear" in names and "wq_pack" in names and len(names) >= 10
    lib = ctypes.CDLL(wqm.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    for s in range(6):
        assert wqm.wq_status_string(s)
    assert wqm.wq_status_string(99) == "unknown status"


@pytest.mark.parametrize("fmt,G", [("int4_sym", 64), ("int4_asym", 128), ("int8_sym", 256),
                                   ("cb4", 0), ("nvfp4", 16), ("mxfp4", 32), ("fp8_e4m3", 128),
                                   ("fp8_e5m2", 64), ("int2_sym", 32), ("int3_sym", 64)])
def test_sizes(fmt, G):
    import synth.workloads as W
    N, K = 4096, 4096
    wb, sb, ab = wqm.wq_packed_sizes(fmt, N, K, G)
    assert wb + sb + ab == W.packed_bytes(fmt, N, K, G if G else 16)
    cb, cs, ca = wqm.wq_canonical_sizes(fmt, N, K, G)
    assert cb == wb and cs == sb
    if fmt == "int4_asym":
        assert ca == 2 * ab


BAD_SHAPES = [
    dict(fmt=10), dict(fmt=-1), dict(fmt="int2_sym", G=16), dict(fmt="int3_sym", G=16), dict(N=0), dict(K=0), dict(N=24), dict(K=96), dict(G=48),
    dict(G=512), dict(fmt="nvfp4", G=32), dict(fmt="mxfp4", G=16), dict(fmt="fp8_e4m3", G=16),
    dict(fmt="fp8_e5m2", G=0), dict(M=-1),
]


@pytest.mark.parametrize("bad", BAD_SHAPES, ids=[str(b) for b in BAD_SHAPES])
def test_linear_rejects_bad_shapes(bad):
    a = dict(fmt="int4_sym", M=4, N=256, K=512, G=64)
    a.update(bad)
    base = 1 << 20
    st = wqm._lib.wq_linear(base, base * 2, base * 3, base * 4, None, a["M"], a["N"], a["K"],
                            wqm._fmt(a["fmt"]), a["G"], base * 5, 0)
    assert st == wqm.WQ_ERR_INVALID_ARG


def test_linear_rejects_null_and_misaligned():
    base = 1 << 20
    f = wqm.FORMATS["int4_asym"]
    # null aux for a format that needs it
    assert wqm._lib.wq_linear(base, base * 2, base * 3, None, None, 4, 256, 512, f, 64, base * 5,
                              0) == wqm.WQ_ERR_INVALID_ARG
    # misaligned x
    assert wqm._lib.wq_linear(base + 2, base * 2, base * 3, base * 4, None, 4, 256, 512, f, 64,
                              base * 5, 0) == wqm.WQ_ERR_ALIGNMENT
    # misaligned output
    assert wqm._lib.wq_linear(base, base * 2, base * 3, base * 4, None, 4, 256, 512, f, 64,
                              base * 5 + 8, 0) == wqm.WQ_ERR_ALIGNMENT
    # output overlapping the activations
    assert wqm._lib.wq_linear(base, base * 2, base * 3, base * 4, None, 4, 256, 512, f, 64,
                              base + 256, 0) == wqm.WQ_ERR_INVALID_ARG


def test_linear_empty_batch_is_noop():
    base = 1 << 20
    st = wqm._lib.wq_linear(base, base * 2, base * 3, None, None, 0, 256, 512,
                            wqm.FORMATS["int4_sym"], 64, base * 5, 0)
    assert st == wqm.WQ_OK


def test_pack_and_quantize_reject_bad_args():
    base = 1 << 20
    f = wqm.FORMATS["cb4"]
    assert wqm._lib.wq_pack(f, 256, 512, 0, base, base, None, base, base, base, 0) == \
        wqm.WQ_ERR_INVALID_ARG
    assert wqm._lib.wq_quantize(wqm.FORMATS["int8_sym"], 256, 500, 64, base, base, base, None, 0) \
        == wqm.WQ_ERR_INVALID_ARG
    assert wqm._lib.wq_dequant(f, 256, 512, 0, None, base, base, base, 0) == wqm.WQ_ERR_INVALID_ARG


def test_lloyd_max_host_matches_oracle(orc):
    """Two independent statements of the Lloyd-Max iteration agree in fp32."""
    c = wqm.wq_lloyd_max_centroids(4)
    _, c32, _, _ = orc.lloyd_max(16)
    assert np.max(np.abs(c.view(np.int32) - c32.view(np.int32))) <= 1
    assert np.all(np.diff(c) > 0)


def test_linear_swiglu_rejects_bad_workspace():
    base = 1 << 20
    f = wqm.FORMATS["int4_sym"]
    M, N, K, G = 64, 256, 512, 64
    args = (base, base * 4, base * 8, None, None, M, N, K, f, G)
    out = base * 64
    ok_ws = base * 32
    need = M * K * 2
    # missing, too small, misaligned, overlapping the input or the output
    assert wqm._lib.wq_linear_swiglu(*args, None, 0, out, 0) == wqm.WQ_ERR_INVALID_ARG
    assert wqm._lib.wq_linear_swiglu(*args, ok_ws, need - 16, out, 0) == wqm.WQ_ERR_INVALID_ARG
    assert wqm._lib.wq_linear_swiglu(*args, ok_ws + 8, need, out, 0) == wqm.WQ_ERR_ALIGNMENT
    assert wqm._lib.wq_linear_swiglu(*args, base + 64, need, out, 0) == wqm.WQ_ERR_INVALID_ARG
    assert wqm._lib.wq_linear_swiglu(*args, out - 64, need, out, 0) == wqm.WQ_ERR_INVALID_ARG
    # the output may not overlap the [up | gate] input (2K values per row)
    assert wqm._lib.wq_linear_swiglu(*args, ok_ws, need, base + M * K * 2, 0) == \
        wqm.WQ_ERR_INVALID_ARG
    # M == 0 is a no-op even without a workspace
    assert wqm._lib.wq_linear_swiglu(base, base * 4, base * 8, None, None, 0, N, K, f, G, None, 0,
                                     out, 0) == wqm.WQ_OK


def test_linear_grouped_rejects_bad_offsets_and_args():
    base = 1 << 20
    f = wqm.FORMATS["int4_sym"]
    N, K, G = 256, 512, 64
    E = 3
    arr = ctypes.c_void_p * E
    w = arr(*[base * (8 + e) for e in range(E)])
    s = arr(*[base * (16 + e) for e in range(E)])

    def call(offs, out=base * 64, g=G):
        o = (ctypes.c_int64 * (E + 1))(*offs)
        return wqm._lib.wq_linear_grouped(base, w, s, None, None, o, E, N, K, f, g, out, 0)

    assert call([1, 2, 3, 4]) == wqm.WQ_ERR_INVALID_ARG        # offsets[0] != 0
    assert call([0, 3, 2, 4]) == wqm.WQ_ERR_INVALID_ARG        # decreasing
    assert call([0, 1, 2, 4], g=48) == wqm.WQ_ERR_INVALID_ARG  # bad group size
    assert call([0, 1, 2, 4], out=base * 64 + 8) == wqm.WQ_ERR_ALIGNMENT
    assert call([0, 0, 0, 0]) == wqm.WQ_OK                     # no rows: nothing launched


def test_addmm_requant_rejections():
    base = 1 << 20
    i8, i4 = wqm.FORMATS["int8_sym"], wqm.FORMATS["int4_sym"]
    N, K, G = 256, 512, 64
    call = wqm._lib.wq_addmm_requant
    assert call(i4, N, K, G, base, base * 8, base * 16, base * 32, 8, 1.0, 1.0, 0, 0, 0) == \
        wqm.WQ_ERR_UNSUPPORTED
    assert call(i8, N, K, G, base, base * 8, base * 16, base * 32, -1, 1.0, 1.0, 0, 0, 0) == \
        wqm.WQ_ERR_INVALID_ARG
    assert call(i8, N, K, G, base + 8, base * 8, base * 16, base * 32, 8, 1.0, 1.0, 0, 0, 0) == \
        wqm.WQ_ERR_ALIGNMENT
    assert call(i8, N, K, G, base, base * 8, None, base * 32, 8, 1.0, 1.0, 0, 0, 0) == \
        wqm.WQ_ERR_INVALID_ARG
    # the weight may not overlap the scales
    assert call(i8, N, K, G, base, base + 64, base * 16, base * 32, 8, 1.0, 1.0, 0, 0, 0) == \
        wqm.WQ_ERR_INVALID_ARG


def test_every_header_call_has_a_binding():
    """The Python binding carries every C name the header declares."""
    missing = [n for n in _declared() if not callable(getattr(wqm, n, None))]
    assert not missing, missing


def test_linear_a8_argument_checks():
    """The activation-quantized linear refuses what it has no kernel for and
    bad workspaces before launching anything (fake, aligned addresses)."""
    base = 1 << 30
    x, w, s, out, ws = base, base * 2, base * 3, base * 4, base * 5
    f8, f4 = wqm.FORMATS["int8_sym"], wqm.FORMATS["int2_sym"]
    M, N, K, G = 64, 256, 1024, 128
    need = wqm.wq_linear_a8_workspace_size(M, K)
    assert need == ((M * K + 255) // 256) * 256 + 4 * M
    lib = wqm._lib
    assert lib.wq_linear_a8(x, w, s, None, M, N, K, f4, G, ws, need, out, None) == \
        wqm.WQ_ERR_UNSUPPORTED
    assert lib.wq_linear_a8(x, w, s, None, M, N, 1088, f8, 64, ws, need * 2, out, None) == \
        wqm.WQ_ERR_UNSUPPORTED                                   # K % 128 != 0
    assert lib.wq_linear_a8(x, w, s, None, M, N, K, f8, G, ws, need - 1, out, None) == \
        wqm.WQ_ERR_INVALID_ARG                                   # workspace too small
    assert lib.wq_linear_a8(x, w, s, None, M, N, K, f8, G, None, need, out, None) == \
        wqm.WQ_ERR_INVALID_ARG
    assert lib.wq_linear_a8(x, w, s, None, M, N, K, f8, G, ws + 8, need, out, None) == \
        wqm.WQ_ERR_ALIGNMENT
    assert lib.wq_linear_a8(x, w, s, None, M, N, K, f8, G, x, need, out, None) == \
        wqm.WQ_ERR_INVALID_ARG                                   # workspace overlaps x
    assert lib.wq_linear_a8(x, w, s, None, M, N, K, f8, 48, ws, need, out, None) == \
        wqm.WQ_ERR_INVALID_ARG                                   # bad group
    assert lib.wq_linear_a8(x, w, s, None, 0, N, K, f8, G, None, 0, out, None) == wqm.WQ_OK
    assert lib.wq_quantize_act_int8(x, M, 1020, ws, ws + M * 1024, None) == \
        wqm.WQ_ERR_INVALID_ARG                                   # K % 8 != 0
    assert lib.wq_quantize_act_int8(x + 8, M, K, ws, ws + M * K, None) == wqm.WQ_ERR_ALIGNMENT
