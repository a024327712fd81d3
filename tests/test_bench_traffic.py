"""bench.py's `roofline.traffic`: the DRAM bytes of one captured prefill GEMM
launch are reported only while the GEMM kernel sources hash to the value
recorded with that capture, so a kernel change turns the figure into null
until the launch is captured again (no GPU needed)."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_is_reported_only_for_the_hashed_sources(monkeypatch):
    h = bench.gemm_sources_sha256()
    monkeypatch.setitem(bench.GEMM_TRAFFIC, "sources_sha256", h)
    assert bench.gemm_traffic() == bench.GEMM_TRAFFIC["bytes"]
    monkeypatch.setitem(bench.GEMM_TRAFFIC, "sources_sha256", "0" * 64)
    assert bench.gemm_traffic() is None


def test_every_listed_source_is_in_the_hash(tmp_path, monkeypatch):
    csrc = os.path.join(tmp_path, "fp8_block_scaled_10_b200", "csrc")
    os.makedirs(csrc)
    for name in bench.GEMM_SOURCES:
        shutil.copy(os.path.join(ROOT, "fp8_block_scaled_10_b200", "csrc", name), csrc)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.gemm_sources_sha256()
    for name in bench.GEMM_SOURCES:
        path = os.path.join(csrc, name)
        with open(path, "rb") as f:
            orig = f.read()
        with open(path, "wb") as f:
            f.write(orig + b"\n")
        assert bench.gemm_sources_sha256() != base, name
        with open(path, "wb") as f:
            f.write(orig)
    assert bench.gemm_sources_sha256() == base
    # every GEMM kernel file of the package is listed
    kernel_files = {"gemm.cuh", "gemm_bs.cuh", "linear.cuh", "sm100.cuh", "quant.cuh", "plan.h", "fp8bs.cu"}
    assert kernel_files <= set(bench.GEMM_SOURCES)
