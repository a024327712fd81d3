"""The GEMM's bounded device waits, made to run out without faulting the GPU.

fp8bs_selftest_gemm_stall withholds one arrival of the first CTA's scale
producer, so that CTA's epilogue waits for a K-block step that never becomes
ready.  The wait must give up after its limit (about 2 s) and record
FP8BS_ERR_TIMEOUT; every role of that CTA then drains its copies and MMAs in
flight, frees its tensor memory and exits.  The host reads the error, and a
normal GEMM on the same context afterwards must still match the oracle.
(The pages show no failure handling; this is the library's own failure
path, tested with a flag that nothing sets instead of a fault.)
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import assert_gemm_close, cuda_codes, cuda_f32, quantized_weight

pytestmark = pytest.mark.gpu


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


def test_withheld_arrival_times_out_and_context_survives():
    from fp8_block_scaled_10_b200 import build
    build.build()
    L = fp8bs.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert fp8bs.device_error() == 0
    M, N, K = 256, 512, 1024
    x = wl.normal_with_outliers(M, K, seed=95, frac=0.01, factor=50.0)
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    qw, sw = quantized_weight(N, K, seed=96)
    a, a_s, w, w_s = cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw)
    nws = fp8bs.gemm_workspace_size(M, N, K)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")

    assert L.fp8bs_selftest_gemm_stall(_vp(a), _vp(a_s), _vp(w), _vp(w_s), M, N, K, _vp(y),
                                       _vp(ws), nws, 0, stream) == fp8bs.ERR_INVALID_ARG
    t0 = time.perf_counter()
    st = L.fp8bs_selftest_gemm_stall(_vp(a), _vp(a_s), _vp(w), _vp(w_s), M, N, K, _vp(y),
                                     _vp(ws), nws, 2, stream)
    assert st == fp8bs.OK, L.fp8bs_last_error_message()
    code = ctypes.c_int(-1)
    assert L.fp8bs_get_device_error(stream, ctypes.byref(code)) == fp8bs.OK
    elapsed = time.perf_counter() - t0
    assert code.value == fp8bs.ERR_TIMEOUT, code.value
    assert elapsed < 30.0, elapsed          # the wait gave up, it did not hang
    assert fp8bs.device_error() == 0        # the error word was read and cleared

    # the same context runs a normal GEMM correctly afterwards
    y2 = fp8bs.fp8_gemm(a, a_s, w, w_s)
    y_ref, bound = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y2, y_ref, bound, "GEMM after the timeout")
    assert fp8bs.device_error() == 0
