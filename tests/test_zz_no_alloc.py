"""fp8bs_fp8_gemm_static_scratch: the GEMM entry point for callers that cannot
allocate device memory (a server that reserves all device memory up front, a
plugin whose host owns the allocator, a C caller without a workspace).  It
keeps its split-K partials in a static device array of the library instead
of a caller workspace.

Checked through the C ABI against fp8bs_fp8_gemm (which is given a torch
workspace) on a split-K problem, for two calls in a row; the second call
reuses the array the first one left behind.  Both entry points run the same
plan, kernels and summation order, so their outputs must agree bit for bit;
both are also held to the GEMM tolerance against the oracle's FP64 product.
Oversize problems must be refused before any launch.  This file is collected
last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import GEMM_ABS_OF_BOUND, GEMM_REL, cuda_codes, cuda_f32, quantized_weight

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 16 * 1024 * 1024   # FP8BS_STATIC_SCRATCH_BYTES in include/fp8bs.h


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_static_scratch_gemm_matches_workspace_gemm():
    from fp8_block_scaled_10_b200 import build
    build.build()
    L = fp8bs.lib()
    M, N, K = 8, 7168, 18432                   # decode down-projection: a split-K plan
    need = fp8bs.gemm_workspace_size(M, N, K)
    assert 0 < need <= STATIC_SCRATCH_BYTES, fp8bs.gemm_plan(M, N, K)

    x = wl.normal_with_outliers(M, K, seed=80, frac=0.01, factor=50.0)
    qa, sa = oracle.act_quant(wl.bf16_bits(x), scale_fmt="ue8m0")
    qw, sw = quantized_weight(N, K, seed=81, scale_fmt="ue8m0")
    a, a_s, w, w_s = cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw)

    # the existing entry point, with a caller-provided workspace
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    y_ws = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    assert L.fp8bs_fp8_gemm(_vp(a), _vp(a_s), _vp(w), _vp(w_s), M, N, K, _vp(y_ws),
                            _vp(ws), need, _stream()) == fp8bs.OK
    y_ref, bound = oracle.gemm(qa, sa, qw, sw)
    tol = GEMM_REL * np.abs(y_ref) + GEMM_ABS_OF_BOUND * bound
    err_ws = np.abs(y_ws.float().cpu().numpy().astype(np.float64) - y_ref)
    assert np.all(err_ws <= tol), "workspace GEMM: %d outputs outside tolerance" % int((err_ws > tol).sum())

    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = L.fp8bs_fp8_gemm_static_scratch(_vp(a), _vp(a_s), _vp(w), _vp(w_s), M, N, K,
                                             _vp(y), _stream())
        assert st == fp8bs.OK, L.fp8bs_last_error_message()
        # same plan and summation order as the workspace call: identical bits
        assert torch.equal(y.view(torch.int16), y_ws.view(torch.int16)), \
            "call %d: %d outputs differ from fp8bs_fp8_gemm" % (call, int((y.view(torch.int16) != y_ws.view(torch.int16)).sum()))
        err = np.abs(y.float().cpu().numpy().astype(np.float64) - y_ref)
        assert np.all(err <= tol), "call %d: %d outputs outside tolerance" % (call, int((err > tol).sum()))
    assert fp8bs.device_error() == 0


def test_static_scratch_gemm_refuses_oversize_problems():
    L = fp8bs.lib()
    for (M, N, K) in [(128, 7168, 18432), (128, 18432, 7168), (256, 7168, 18432), (512, 4096, 18432),
                      (1024, 2048, 18432), (100, 65536, 16384)]:
        if fp8bs.gemm_workspace_size(M, N, K) > STATIC_SCRATCH_BYTES:
            break
    else:
        pytest.skip("no candidate shape needs more split-K scratch than the static array")
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    st = L.fp8bs_fp8_gemm_static_scratch(_vp(dummy), _vp(dummy), _vp(dummy), _vp(dummy),
                                         M, N, K, _vp(dummy), _stream())
    assert st == fp8bs.ERR_WORKSPACE
    assert b"static scratch" in L.fp8bs_last_error_message()
