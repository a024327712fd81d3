"""The grouped GEMM's unit decoding, checked on the CPU: tests/grouped_check.cu
includes the kernel header and runs its __host__ __device__ grouped_unit over
the group table layout the kernel builds, for many expert layouts (empty
groups, offsets past M, out-of-contract offsets the kernel clamps).  In
contract, every row of every group is computed exactly once per n tile and
no other row at all; out of contract, every unit still stays inside [0, M)
(nvcc compiles the host side; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_grouped_units_cover_each_group_row_once(tmp_path):
    exe = tmp_path / "grouped_check"
    cmd = [NVCC, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "fp8_block_scaled_10_b200", "csrc"),
           os.path.join(HERE, "grouped_check.cu"), "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
