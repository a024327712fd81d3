"""The GEMM's dense tile order (bands of n tiles, m fastest inside a band)
and the transposing kernels' tile order (groups of 8 row bands), checked on
the CPU: tests/tile_order_check.cu includes the kernel headers and runs their
__host__ __device__ tile_mn and tile_coords over many shapes (no GPU needed;
nvcc compiles the host side)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_tile_order_is_a_bijection(tmp_path):
    exe = tmp_path / "tile_order_check"
    cmd = [NVCC, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "fp8_block_scaled_10_b200", "csrc"),
           os.path.join(HERE, "tile_order_check.cu"), "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
