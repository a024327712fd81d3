"""fp8_gemm with an FP32 output ("DeepSeek-V3: How Selective FP8 Stays
Stable", "Lower precision is a constrained budget": the FP8 GEMMs' outputs
may be BF16 or FP32).

The FP32 y is the kernel's accumulator itself, so against the oracle's FP64
product it carries only the accumulation error: |dy| <= 2^-23 |y_ref| +
1e-3 sum_k |a_k w_k| (the bf16 tolerance with its output-rounding term
replaced by fp32's).  And since the bf16 entry point rounds the same
accumulator, in the same order, under the same launch plan, bf16_rne(y_f32)
must equal its output bit for bit.  Shapes cover the TMA store path
(N % 4 == 0), the direct stores (N % 4 != 0), K splits with their FP32
reduction (decode M), the split tail and both scale formats."""
import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import GEMM_ABS_OF_BOUND, cuda_codes, cuda_f32, quantized_weight

pytestmark = pytest.mark.gpu

F32_REL = 2.0 ** -23


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_block_scaled_10_b200 import build
    build.build()
    yield
    assert fp8bs.device_error() == 0


def _check_f32(y, y_ref, bnd, what):
    yv = y.cpu().numpy().astype(np.float64)
    err = np.abs(yv - y_ref)
    tol = F32_REL * np.abs(y_ref) + GEMM_ABS_OF_BOUND * bnd
    bad = ~(err <= tol)
    assert not bad.any(), "%s: %d outside, first %s" % (what, int(bad.sum()), np.argwhere(bad)[:3])


@pytest.mark.parametrize("fmt", [None, "ue8m0"])
@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512), (1, 256, 128), (129, 130, 256), (300, 1280, 1024), (200, 131, 384),
    (8, 7168, 18432 // 4), (64, 18432 // 8, 7168), (1200, 4000, 4096),
])
def test_f32_output(M, N, K, fmt):
    x = wl.normal_with_outliers(M, K, seed=M + 7 * N + K, frac=0.01, factor=50.0)
    qa, sa = oracle.act_quant(wl.bf16_bits(x), scale_fmt=fmt)
    qw, sw = quantized_weight(N, K, seed=M + 5 * N, scale_fmt=fmt)
    args = (cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw))
    y32 = fp8bs.fp8_gemm(*args, scale_fmt=fmt, out_dtype=torch.float32)
    y16 = fp8bs.fp8_gemm(*args, scale_fmt=fmt)
    assert y32.dtype == torch.float32 and y32.shape == (M, N)
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    plan = fp8bs.gemm_plan(M, N, K)
    _check_f32(y32, y_ref, bnd, "f32 gemm %dx%dx%d %s [%s]" % (M, N, K, fmt, plan))
    # the bf16 output is the same accumulator rounded to nearest even
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y16.view(torch.int16)), plan


def test_f32_output_not_rounded_to_bf16():
    """Most FP32 outputs carry bits below bf16 precision (an FP32 y that went
    through bf16 would have none)."""
    M, N, K = 256, 512, 1024
    x = wl.normal_with_outliers(M, K, seed=3, frac=0.01, factor=50.0)
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    qw, sw = quantized_weight(N, K, seed=4)
    y32 = fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw),
                         out_dtype=torch.float32)
    low = (y32.view(torch.int32) & 0xFFFF) != 0
    assert low.float().mean().item() > 0.9
