"""The dense GEMM planner, checked on the CPU: tests/plan_check.cu includes
the planner header and runs every plan through the kernels' own unit decoding
(gemm::dense_unit, __host__ __device__), so a plan whose units skip or repeat
a (tile, K block), or whose split-tail slots disagree with the tail
reduction, fails here without a GPU (nvcc compiles the host side)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_every_plan_covers_each_tile_and_k_block_once(tmp_path):
    exe = tmp_path / "plan_check"
    cmd = [NVCC, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "fp8_block_scaled_10_b200", "csrc"),
           os.path.join(HERE, "plan_check.cu"), "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
