"""The few-token table kernel's shared-memory layout rules, checked on the host.

tests/host/lut_layout_check.cu includes the kernel header and checks, for every K up to 65536
and a range of token counts, tiles and ring sizes: the strides that keep the kernel's shared
loads free of bank conflicts (tile rows 8 mod 32 words, scale rows 4 mod 32 floats), the
16-byte alignment that the bulk copies and quad loads need, and that every region of the
layout holds what the kernel writes there without overlapping the next one.
"""
import os
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def test_lut_layout_rules():
    src = os.path.join(ROOT, "tests", "host", "lut_layout_check.cu")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "lut_layout_check")
        try:
            subprocess.run([nvcc(), "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                            "-I", os.path.join(ROOT, "include"),
                            "-I", os.path.join(ROOT, "bit_nf4_quantized_quantize_b200", "csrc"),
                            "-o", exe, src], check=True, capture_output=True, timeout=600)
        except FileNotFoundError:
            pytest.skip("nvcc not available")
        out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
