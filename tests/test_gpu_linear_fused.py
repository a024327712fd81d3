"""The fused FP8 linear layer: act_quant and the GEMM in one launch.

When the GEMM's tiles leave SMs idle, fp8bs_fp8_linear_fused gives those SMs
the quantization of x and lets the GEMM consume each quantized chunk as soon
as its ready flag is set ("Understanding Dynamic and Static Activation
Quantization Schemes in DeepSeek-V3", "How Dynamic Activation Quantization
Works": the linear layer calls act_quant in its forward pass).  Checked here:
q and s bit for bit against the oracle's act_quant, y against the oracle's
FP64 GEMM on those codes, nothing written outside q, s and y, and the same
q / s as the two-launch form on identical inputs.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import assert_gemm_close, cuda_codes, cuda_f32, f32bits, quantized_weight, sample_rows, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_block_scaled_10_b200 import build
    build.build()
    torch.cuda.init()
    yield
    assert fp8bs.device_error() == 0


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _sms148():
    return fp8bs.gemm_plan(4096, 4096, 1024).find("sms=148") >= 0


def _run_two_launches(x, qw, sw):
    """The unfused form: fp8bs_act_quant, then fp8bs_fp8_gemm (C ABI)."""
    L = fp8bs.lib()
    M, K = x.shape
    N = qw.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    x_d = x.cuda()
    w_d, sw_d = cuda_codes(qw).view(torch.uint8), cuda_f32(sw)
    q = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    s = torch.empty(M, K // 128, dtype=torch.float32, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nws = int(L.fp8bs_gemm_workspace_size(M, N, K))
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    assert L.fp8bs_act_quant(_vp(x_d), 0, M, K, 128, 0, _vp(q), _vp(s), stream) == fp8bs.OK
    assert L.fp8bs_fp8_gemm(_vp(q), _vp(s), _vp(w_d), _vp(sw_d), M, N, K, _vp(y), _vp(ws), nws,
                            stream) == fp8bs.OK
    torch.cuda.synchronize()
    return q, s, y


def _run_linear(x, qw, sw, fmt):
    """fp8bs_fp8_linear_fused through the C ABI with canaries around q, s and y."""
    L = fp8bs.lib()
    M, K = x.shape
    N = qw.shape[0]
    x_d = x.cuda()
    w_d, sw_d = cuda_codes(qw).view(torch.uint8), cuda_f32(sw)
    qbig = torch.full((M + 2, K), 0x5A, dtype=torch.uint8, device="cuda")
    sbig = torch.full((M + 2, K // 128), -3.0, dtype=torch.float32, device="cuda")
    ybig = torch.full((M + 2, N), -7.0, dtype=torch.bfloat16, device="cuda")
    q, s, y = qbig[1:M + 1], sbig[1:M + 1], ybig[1:M + 1]
    nws = int(L.fp8bs_linear_workspace_size(M, N, K))
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    st = L.fp8bs_fp8_linear_fused(_vp(x_d), M, K, 1 if fmt else 0, _vp(w_d), _vp(sw_d), N,
                                  _vp(y), _vp(q), _vp(s), _vp(ws), nws,
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == fp8bs.OK, L.fp8bs_last_error_message()
    torch.cuda.synchronize()
    for big, fill in ((qbig, 0x5A), (sbig, -3.0), (ybig, -7.0)):
        assert torch.all(big[0] == fill) and torch.all(big[M + 1] == fill), "canary row overwritten"
    return q, s, y


@pytest.mark.parametrize("fmt", [None, "ue8m0"])
@pytest.mark.parametrize("M,N,K", [(300, 512, 1024), (129, 256, 512), (1000, 576, 2048)])
def test_fused_linear_matches_oracle(M, N, K, fmt):
    plan = fp8bs.linear_plan(M, N, K)
    x = wl.normal_with_outliers(M, K, seed=M + K, frac=0.01, factor=50.0)
    qw, sw = quantized_weight(N, K, seed=N + K, scale_fmt=fmt)
    q, s, y = _run_linear(x, qw, sw, fmt)
    qa, sa = oracle.act_quant(wl.bf16_bits(x), scale_fmt=fmt)
    assert np.array_equal(u8(q), qa), plan
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(sa)), plan
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "fused linear " + plan)
    assert fp8bs.device_error() == 0


def test_fused_and_two_launch_forms_agree():
    """Same inputs through both forms: identical q and s, y within tolerance of
    each other's oracle product (the tile plans differ)."""
    M, N, K = 4096, 576, 7168
    plan = fp8bs.linear_plan(M, N, K)
    if _sms148():
        assert "fused: bn=" in plan, plan   # a fused launch exists for this shape
    x = wl.heavy_tailed_channels(M, K, seed=61)
    qw, sw = quantized_weight(N, K, seed=62)
    q1, s1, y1 = _run_linear(x, qw, sw, None)
    q2, s2, y2 = _run_two_launches(x, qw, sw)
    assert torch.equal(q1, q2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    assert np.array_equal(u8(q1), qa)
    rows = sample_rows(M, 16, seed=63)
    y_ref, bnd = oracle.gemm(qa[rows], sa[rows], qw, sw)
    idx = torch.from_numpy(rows).cuda()
    assert_gemm_close(y1[idx], y_ref, bnd, "fused " + plan)
    assert_gemm_close(y2[idx], y_ref, bnd, "two launches")
    assert fp8bs.device_error() == 0


def test_fused_linear_is_repeatable():
    """Back-to-back fused calls reuse the workspace flags (reset each call)."""
    M, N, K = 1000, 576, 2048
    x = wl.normal_with_outliers(M, K, seed=71, frac=0.01, factor=50.0)
    qw, sw = quantized_weight(N, K, seed=72)
    outs = [_run_linear(x, qw, sw, None) for _ in range(3)]
    for q, s, y in outs[1:]:
        assert torch.equal(q, outs[0][0]) and torch.equal(y.view(torch.int16), outs[0][2].view(torch.int16))


def test_fused_linear_refuses_what_it_cannot_run():
    """No fused launch at decode-sized M or when the tiles fill the GPU, and a
    workspace too small for the chunk flags is refused before any launch."""
    L = fp8bs.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    d = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    for (M, N, K) in [(64, 576, 1024), (4096, 18432, 1024)]:
        st = L.fp8bs_fp8_linear_fused(_vp(d), M, K, 0, _vp(d), _vp(d), N, _vp(d), _vp(d), _vp(d),
                                      _vp(ws), ws.numel(), stream)
        assert st == fp8bs.ERR_UNSUPPORTED, (M, N, L.fp8bs_last_error_message())
    st = L.fp8bs_fp8_linear_fused(_vp(d), 1000, 2048, 0, _vp(d), _vp(d), 576, _vp(d), _vp(d),
                                  _vp(d), _vp(ws), 64, stream)
    assert st == fp8bs.ERR_WORKSPACE


def test_python_binding_matches_two_launch_form():
    """fp8bs.fp8_linear_fused (the binding) against fp8bs.fp8_linear on the
    same inputs: identical q and s; y within tolerance of the oracle."""
    M, N, K = 1000, 576, 2048
    x = wl.normal_with_outliers(M, K, seed=81, frac=0.01, factor=50.0).cuda()
    qw, sw = quantized_weight(N, K, seed=82)
    w_d, sw_d = cuda_codes(qw), cuda_f32(sw)
    y1, q1, s1 = fp8bs.fp8_linear_fused(x, w_d, sw_d, return_quant=True)
    y2, q2, s2 = fp8bs.fp8_linear(x, w_d, sw_d, return_quant=True)
    assert torch.equal(q1.view(torch.uint8), q2.view(torch.uint8))
    assert torch.equal(s1.view(torch.int32), s2.view(torch.int32))
    qa, sa = oracle.act_quant(wl.bf16_bits(x.cpu()))
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y1, y_ref, bnd, "fp8_linear_fused binding")
    with pytest.raises(fp8bs.Fp8bsError):
        fp8bs.fp8_linear_fused(x[:64], w_d, sw_d)     # decode-sized M: no fused launch
    assert fp8bs.device_error() == 0
