"""The packed weight layout, checked on the host: compiles tests/layout_check.cu
(host code only, nvcc) and runs it.  Every format's element -> (byte, bit)
map must be a bijection onto the packed bits, and the nibble / 2-bit field
orders must hand each fragment register the elements the tensor-core step
expects."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc (host compilation only)")
def test_packed_layout_bijection_and_fragments(tmp_path):
    exe = str(tmp_path / "layout_check")
    subprocess.run(["nvcc", "-std=c++17", "-x", "cu", "-o", exe,
                    os.path.join(HERE, "layout_check.cu")], check=True, capture_output=True,
                   timeout=300)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "FAIL" not in out.stdout
