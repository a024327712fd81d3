"""The GEMM kernels' static resource budgets (shared memory, control block,
TMEM columns, swizzle alignment, warp register split, and the decode path's
128-row A over-read staying inside the allocation), checked by static_assert
in a host build of the kernel headers: tests/budget_check.cu (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_every_launched_configuration_fits_its_budgets(tmp_path):
    exe = tmp_path / "budget_check"
    cmd = [NVCC, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "fp8_block_scaled_10_b200", "csrc"),
           os.path.join(HERE, "budget_check.cu"), "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
