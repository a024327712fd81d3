"""fp8_gemm_quant, the GEMM with an FP8 output: the bf16 y it also returns is
within the GEMM tolerance of the oracle's FP64 product, and its q / s are
bit-identical to the oracle's act_quant of that bf16 y (1x128 blocks along
N, scale_fmt None or ue8m0), every element."""
import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import assert_gemm_close, cuda_codes, cuda_f32, f32bits, quantized_weight, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_block_scaled_10_b200 import build
    build.build()
    yield
    assert fp8bs.device_error() == 0


@pytest.mark.parametrize("out_fmt", [None, "ue8m0"])
@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512), (1, 256, 128), (300, 1280, 1024), (64, 2048, 2048), (1000, 384, 7168),
    (513, 128, 256),
])
def test_fp8_output_matches_act_quant_of_y(M, N, K, out_fmt):
    x = wl.normal_with_outliers(M, K, seed=M + N + K, frac=0.01, factor=50.0)
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    qw, sw = quantized_weight(N, K, seed=M + 3 * N)
    args = (cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw))
    q, s, y = fp8bs.fp8_gemm_quant(*args, out_scale_fmt=out_fmt, return_y=True)
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "fp8-output gemm %dx%dx%d" % (M, N, K))
    yb = y.view(torch.int16).cpu().numpy().view(np.uint16)
    q_ref, s_ref = oracle.act_quant(yb, scale_fmt=out_fmt)
    assert q.shape == (M, N) and s.shape == (M, N // 128)
    assert np.array_equal(u8(q), q_ref)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))
    # without the bf16 y the codes and scales are the same
    q2, s2 = fp8bs.fp8_gemm_quant(*args, out_scale_fmt=out_fmt)
    assert torch.equal(q2.view(torch.uint8), q.view(torch.uint8))
    assert torch.equal(s2.view(torch.int32), s.view(torch.int32))


def test_fp8_output_prefill_shape_sampled():
    """M=4096, K=7168, N=18432 (ue8m0 output, as a following decode-style
    layer would take it): q / s of every element against the oracle's
    act_quant of the returned y."""
    M, K, N = 4096, 7168, 18432
    x = wl.heavy_tailed_channels(M, K, seed=90)
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    qw, sw = quantized_weight(N, K, seed=91)
    q, s, y = fp8bs.fp8_gemm_quant(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw),
                                   out_scale_fmt="ue8m0", return_y=True)
    yb = y.view(torch.int16).cpu().numpy().view(np.uint16)
    q_ref, s_ref = oracle.act_quant(yb, scale_fmt="ue8m0")
    assert np.array_equal(u8(q), q_ref)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))
