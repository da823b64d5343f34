"""The remainder-corrected quotient behind every UE element and scale code.

The quantizer never divides on its common path: it forms fp32(y / S) from the
correctly rounded reciprocal of S with one remainder correction (Markstein's
division theorem).  tests/cuda/quotient_check.cu compiles the library's own
device header and compares that sequence bit for bit with IEEE division:
exhaustively for every bf16 significand against every fp32 significand (the
whole unrotated path), at the fp32 significands where the first product is
furthest off, on random fp32 pairs, and for signed zeros.
"""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "microscaling_fp4_quantization_block_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "cuda", "quotient_check.cu")


@pytest.mark.gpu
def test_remainder_corrected_quotient_is_ieee_division():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
    exe = os.path.join(ROOT, "_build", "quotient_check")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-fmad=false",
                    "-I", CSRC, SRC, "-o", exe], check=True, capture_output=True, text=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=300).stdout
    rows = {line.split()[0]: (int(line.split()[1]), int(line.split()[2])) for line in out.strip().splitlines()}
    assert rows["bf16_all"][0] == 5 * (1 << 23) * 256
    assert rows["fp32_edges"][0] == 2 * (1 << 23) * 2048
    for name, (count, bad) in rows.items():
        assert count > 0 and bad == 0, (name, count, bad)
