"""The training GEMMs' operands and the row-scaled GEMM on the GPU ("DeepSeek-V3:
How Selective FP8 Stays Stable", "Lower precision is a constrained budget":
forward, activation-gradient and weight-gradient GEMMs all in FP8, weight
gradients in FP32), against the oracle.

* fp8_transpose: codes and block scales, byte for byte (tiled and element-wise
  paths, ragged tiles, the full dense weight [18432, 7168]).
* act_quant_transposed: q and s byte for byte against act_quant of x^T, both
  scale formats and input dtypes, up to the prefill activation [4096, 7168].
* fp8_gemm_rowwise: per-row scales on both operands, within the GEMM
  tolerance (bf16 output) or its fp32 form (fp32 output), for both kernels,
  K splits and ragged edges; on the weight-gradient shape of the dense layer
  (dW [18432, 7168] over 4096 tokens) on sampled rows.
* The activation-gradient GEMM dx = dy W as fp8_gemm(dy, W^T)."""
import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import (GEMM_ABS_OF_BOUND, assert_gemm_close, cuda_codes, cuda_f32, f32bits,
                   quantized_weight, sample_rows, u8)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_block_scaled_10_b200 import build
    build.build()
    yield
    assert fp8bs.device_error() == 0


def _np_input(x):
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view(np.uint16)
    return x.numpy()


# --------------------------------------------------------------------------
# fp8_transpose
# --------------------------------------------------------------------------

@pytest.mark.parametrize("R,C,block", [
    (256, 384, 128), (128, 16, 128), (144, 272, 64), (300, 200, 128), (7, 5, 32), (640, 96, 256),
])
def test_fp8_transpose_matches_oracle(R, C, block):
    codes = wl.e4m3_codes(R, C, seed=R + C).numpy()
    s = wl.uniform((-(-R // block), -(-C // block)), 1e-5, 1e-3, seed=R).numpy()
    qt_ref, st_ref = oracle.fp8_transpose(codes, s, block)
    qt, st = fp8bs.fp8_transpose(torch.from_numpy(codes).cuda(), torch.from_numpy(s).cuda(), block)
    assert np.array_equal(u8(qt), qt_ref)
    assert np.array_equal(f32bits(st.cpu().numpy()), f32bits(st_ref))


def test_fp8_transpose_full_weight():
    """The dense up-projection weight [18432, 7168] and its [144, 56] scales."""
    R, C = 18432, 7168
    codes = wl.e4m3_codes(R, C, seed=30)
    s = wl.uniform((144, 56), 1e-5, 1e-3, seed=31)
    qt, st = fp8bs.fp8_transpose(codes.cuda(), s.cuda())
    assert torch.equal(qt.view(torch.uint8).cpu(), codes.T.contiguous())
    assert torch.equal(st.cpu(), s.T.contiguous())


# --------------------------------------------------------------------------
# act_quant_transposed
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [None, "ue8m0"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("R,C", [(128, 8), (256, 200), (384, 1000), (512, 7168)])
def test_act_quant_transposed_matches_oracle(R, C, dtype, fmt):
    x = wl.normal_with_outliers(R, C, seed=R + C, frac=0.01, factor=50.0, dtype=dtype)
    x[:128, 3] = 0                                    # an all-zero column block
    q_ref, s_ref = oracle.act_quant_transposed(_np_input(x), scale_fmt=fmt)
    q, s = fp8bs.act_quant_transposed(x.cuda(), 128, fmt)
    assert q.shape == (C, R) and s.shape == (C, R // 128)
    assert np.array_equal(u8(q), q_ref)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))


def test_act_quant_transposed_prefill_activation():
    """x bf16 [4096, 7168] with heavy-tailed channels, every byte."""
    x = wl.heavy_tailed_channels(4096, 7168, seed=60)
    q_ref, s_ref = oracle.act_quant_transposed(_np_input(x))
    q, s = fp8bs.act_quant_transposed(x.cuda())
    assert np.array_equal(u8(q), q_ref)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))


# --------------------------------------------------------------------------
# fp8_gemm_rowwise (weight gradient)
# --------------------------------------------------------------------------

def _rowwise_case(M, N, K, seed, fmt):
    """a [M, K] and b [N, K] quantized 1 x 128 along K (as act_quant_transposed
    leaves dy^T and x^T)."""
    a = wl.normal_with_outliers(M, K, seed=seed, frac=0.01, factor=30.0)
    b = wl.normal_with_outliers(N, K, seed=seed + 1, frac=0.01, factor=30.0)
    qa, sa = oracle.act_quant(wl.bf16_bits(a), scale_fmt=fmt)
    qb, sb = oracle.act_quant(wl.bf16_bits(b), scale_fmt=fmt)
    return qa, sa, qb, sb


def _check_f32(y, y_ref, bnd, what):
    yv = y.cpu().numpy().astype(np.float64)
    tol = 2.0 ** -23 * np.abs(y_ref) + GEMM_ABS_OF_BOUND * bnd
    bad = ~(np.abs(yv - y_ref) <= tol)
    assert not bad.any(), "%s: %d outside, first %s" % (what, int(bad.sum()), np.argwhere(bad)[:3])


@pytest.mark.parametrize("fmt", [None, "ue8m0"])
@pytest.mark.parametrize("M,N,K", [
    (128, 256, 128), (130, 200, 256), (300, 384, 1024), (1000, 576, 512), (64, 2048, 4096),
    (1200, 4000, 1024),
])
def test_gemm_rowwise_matches_oracle(M, N, K, fmt):
    qa, sa, qb, sb = _rowwise_case(M, N, K, seed=M + 3 * N + K, fmt=fmt)
    args = (cuda_codes(qa), cuda_f32(sa), cuda_codes(qb), cuda_f32(sb))
    y_ref, bnd = oracle.gemm(qa, sa, qb, sb, w_scales="row")
    y32 = fp8bs.fp8_gemm_rowwise(*args, scale_fmt=fmt)
    _check_f32(y32, y_ref, bnd, "rowwise f32 %dx%dx%d %s" % (M, N, K, fmt))
    y16 = fp8bs.fp8_gemm_rowwise(*args, scale_fmt=fmt, out_dtype=torch.bfloat16)
    assert_gemm_close(y16, y_ref, bnd, "rowwise bf16 %dx%dx%d %s" % (M, N, K, fmt))
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16))


@pytest.mark.parametrize("fmt", [None, "ue8m0"])
def test_weight_gradient_dense_layer(fmt):
    """dW = dy^T x for the dense up-projection over 4096 tokens: dy [4096,
    18432], x [4096, 7168] -> dW [18432, 7168] fp32, through
    act_quant_transposed and fp8_gemm_rowwise, on sampled rows of dW."""
    T, N, K = 4096, 18432, 7168
    dy = wl.normal_with_outliers(T, N, seed=80, frac=0.001, factor=20.0) * 1e-3
    x = wl.heavy_tailed_channels(T, K, seed=81)
    qd, sd = fp8bs.act_quant_transposed(dy.cuda(), 128, fmt)
    qx, sx = fp8bs.act_quant_transposed(x.cuda(), 128, fmt)
    dw = fp8bs.fp8_gemm_rowwise(qd, sd, qx, sx, scale_fmt=fmt)
    rows = sample_rows(N, 24, seed=82)
    qd_ref, sd_ref = oracle.act_quant_transposed(_np_input(dy.to(torch.bfloat16)), scale_fmt=fmt)
    qx_ref, sx_ref = oracle.act_quant_transposed(_np_input(x), scale_fmt=fmt)
    assert np.array_equal(u8(qd)[rows], qd_ref[rows])
    y_ref, bnd = oracle.gemm(qd_ref[rows], sd_ref[rows], qx_ref, sx_ref, w_scales="row")
    _check_f32(dw[torch.from_numpy(rows).cuda()], y_ref, bnd, "dW %s" % fmt)


def test_activation_gradient_through_transposed_weight():
    """dx = dy W for W [N, K] = [2304, 1024]: fp8_gemm(dy, W^T) with W^T from
    fp8_transpose, against the oracle on the same operands."""
    T, N, K = 512, 2304, 1024
    dy = wl.normal_with_outliers(T, N, seed=90, frac=0.01, factor=30.0)
    qd, sd = oracle.act_quant(wl.bf16_bits(dy))
    qw, sw = quantized_weight(N, K, seed=91)
    qwt, swt = fp8bs.fp8_transpose(cuda_codes(qw), cuda_f32(sw))
    dx = fp8bs.fp8_gemm(cuda_codes(qd), cuda_f32(sd), qwt, swt)
    qwt_ref, swt_ref = oracle.fp8_transpose(qw, sw)
    y_ref, bnd = oracle.gemm(qd, sd, qwt_ref, swt_ref)
    assert_gemm_close(dx, y_ref, bnd, "dgrad")
