"""The kernels' division by a per-launch invariant divisor (the row index of
the static quantizer and of the dequantizer), checked on the CPU against
integer division: tests/divide_check.cu includes the kernel header and runs
its __host__ __device__ div_invariant with the host-side invariant_div over
thousands of divisors and every 32-bit n for one of them (nvcc compiles the
host side; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_invariant_division_equals_integer_division(tmp_path):
    exe = tmp_path / "divide_check"
    cmd = [NVCC, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "fp8_block_scaled_10_b200", "csrc"),
           os.path.join(HERE, "divide_check.cu"), "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
