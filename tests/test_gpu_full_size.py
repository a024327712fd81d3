"""Every output of the full-size prefill GEMMs, against a library matmul.

The oracle's FP64 GEMM is too slow for all 75M outputs of a prefill shape, so
the sampled-row parity tests cover it; this test adds a check of every output
through a property that holds at any size: the operands are quantized by the
CPU oracle, dequantized with torch's own float8 cast and the scales, and
multiplied by torch (cuBLAS, FP32, TF32 off).  Against that product the
kernel's bf16 y must stay within |dy| <= 4e-3 |y_ref| + 2e-3 B, with
B = |A_hat| |W_hat|^T: the GEMM tolerance's 1e-3 B for the kernel's FP32
accumulation plus as much again for the library's (both well under 1e-3 B in
practice for K <= 18432)."""
import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import cuda_codes, cuda_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_block_scaled_10_b200 import build
    build.build()
    yield
    assert fp8bs.device_error() == 0


def _dequant(q, s, rows_per_scale):
    """e4m3 codes (device uint8) times their block scales, as float32."""
    v = q.view(torch.float8_e4m3fn).float()
    sc = s.repeat_interleave(128, dim=1)[:, : q.shape[1]]
    if rows_per_scale > 1:
        sc = sc.repeat_interleave(rows_per_scale, dim=0)[: q.shape[0]]
    return v * sc


@pytest.mark.parametrize("K,N", [(7168, 18432), (18432, 7168)])
def test_prefill_every_output_against_library_matmul(K, N):
    M = wl.PREFILL_M
    x = wl.heavy_tailed_channels(M, K, seed=K + N)
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    qw, sw = oracle.weight_quant(wl.weight_f32(N, K, seed=K + N + 1).numpy())
    a, a_s, w, w_s = cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw)
    y = fp8bs.fp8_gemm(a, a_s, w, w_s).float()
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        a_hat = _dequant(a.view(torch.uint8), a_s, 1)
        w_hat = _dequant(w.view(torch.uint8), w_s, 128)
        y_ref = a_hat @ w_hat.T
        bound = a_hat.abs() @ w_hat.abs().T
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    tol = 4e-3 * y_ref.abs() + 2e-3 * bound
    bad = (y - y_ref).abs() > tol
    n_bad = int(bad.sum().item())
    assert n_bad == 0, "%d of %d outputs outside tolerance" % (n_bad, bad.numel())
