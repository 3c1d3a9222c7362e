"""The base-s chunk conversions of the CUDA library (gq_entropy.cuh is plain C++ on 32-bit
integers) compiled for the CPU and checked exhaustively against plain digit arithmetic; no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_swar_conversions_exhaustive(tmp_path):
    exe = str(tmp_path / "swar_check")
    inc = os.path.join(ROOT, "gradient_quantization_communication_b200", "csrc")
    src = os.path.join(ROOT, "tests", "entropy_swar_check.cpp")
    r = subprocess.run(["g++", "-O2", "-std=c++17", "-I" + inc, src, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "chunks done bad=0" in r.stdout
