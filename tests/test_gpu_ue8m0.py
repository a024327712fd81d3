"""Parity of the block-scaled (ue8m0) GEMM path with the CPU oracle.

fp8_gemm_ue8m0 / fp8_linear_ue8m0 / fp8_gemm_grouped_ue8m0 take power-of-two
scales (scale_fmt "ue8m0" for activations and weights) and let the tensor
core apply them.  Results are held to the same tolerance as fp8_gemm:
|dy| <= 4e-3 |y_ref| + 1e-3 sum_k |a_k w_k| against the oracle's FP64 result.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import assert_gemm_close, cuda_codes, cuda_f32, quantized_weight, sample_rows, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_block_scaled_10_b200 import build
    build.build()
    torch.cuda.init()
    yield
    assert fp8bs.device_error() == 0


def _case(M, N, K, seed, heavy=False):
    if heavy:
        x = wl.heavy_tailed_channels(M, K, seed=seed)
    else:
        x = wl.normal_with_outliers(M, K, seed=seed, frac=0.01, factor=50.0)
    qa, sa = oracle.act_quant(wl.bf16_bits(x), scale_fmt="ue8m0")
    qw, sw = quantized_weight(N, K, seed=seed + 1, scale_fmt="ue8m0")
    return x, qa, sa, qw, sw


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512), (1, 256, 128), (127, 576, 512), (129, 130, 256), (300, 384, 1024),
    (256, 512, 7168), (513, 1280, 384), (64, 2048, 2048), (2, 18432, 256), (200, 136, 128),
    # 160 tiles on 148 SMs: the last wave's tiles split along K, ragged edges
    (1200, 4000, 4096),
])
def test_gemm_ue8m0_shapes(M, N, K):
    x, qa, sa, qw, sw = _case(M, N, K, seed=M + 2 * N + K)
    y = fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw), scale_fmt="ue8m0")
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "ue8m0 gemm %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("K,N", wl.DECODE_KN)
@pytest.mark.parametrize("M", wl.DECODE_M)
def test_gemm_ue8m0_decode_full(M, K, N):
    """The decode shapes (ue8m0 scales by definition), every output."""
    x, qa, sa, qw, sw = _case(M, N, K, seed=M * 5 + K)
    y = fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw), scale_fmt="ue8m0")
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "ue8m0 decode M=%d K=%d N=%d (%s)" % (M, K, N, fp8bs.gemm_plan(M, N, K)))


@pytest.mark.parametrize("K,N", wl.PREFILL_KN)
def test_fp8_linear_ue8m0_prefill(K, N):
    M = wl.PREFILL_M
    x = wl.heavy_tailed_channels(M, K, seed=140 + K)
    qw, sw = quantized_weight(N, K, seed=141 + N, scale_fmt="ue8m0")
    y, q, s = fp8bs.fp8_linear(x.cuda(), cuda_codes(qw), cuda_f32(sw), scale_fmt="ue8m0",
                               weight_scale_fmt="ue8m0", return_quant=True)
    qa, sa = oracle.act_quant(wl.bf16_bits(x), scale_fmt="ue8m0")
    assert np.array_equal(u8(q), qa)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), sa.view(np.uint32))
    rows = sample_rows(M, 12, seed=K + N + 1)
    y_ref, bnd = oracle.gemm(qa[rows], sa[rows], qw, sw)
    assert_gemm_close(y[torch.from_numpy(rows).cuda()], y_ref, bnd, "ue8m0 prefill K=%d N=%d" % (K, N))


def _grouped(counts, N, K, seed):
    G = len(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    Mt = int(offs[-1])
    x = wl.normal_with_outliers(max(Mt, 1), K, seed=seed, frac=0.001, factor=20.0)[:Mt]
    qa, sa = oracle.act_quant(wl.bf16_bits(x), scale_fmt="ue8m0")
    qws, sws = zip(*[quantized_weight(N, K, seed=seed + 1 + g, scale_fmt="ue8m0") for g in range(G)])
    return offs, qa, sa, np.stack(qws), np.stack(sws)


def test_grouped_ue8m0_small_ragged():
    counts = [0, 1, 130, 255, 64, 0, 300]
    offs, qa, sa, qw, sw = _grouped(counts, 384, 256, seed=160)
    y = fp8bs.fp8_gemm_grouped(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw),
                               torch.from_numpy(offs).cuda(), scale_fmt="ue8m0")
    for g in range(len(counts)):
        lo, hi = offs[g], offs[g + 1]
        if hi > lo:
            y_ref, bnd = oracle.gemm(qa[lo:hi], sa[lo:hi], qw[g], sw[g])
            assert_gemm_close(y[lo:hi], y_ref, bnd, "ue8m0 group %d" % g)


def test_grouped_ue8m0_expert_config_sampled():
    counts = wl.expert_counts(wl.EXPERT_TOKENS * wl.EXPERT_TOPK, wl.EXPERTS, seed=170).numpy()
    offs, qa, sa, qw, sw = _grouped(counts, wl.EXPERT_FFN, wl.HIDDEN, seed=171)
    y = fp8bs.fp8_gemm_grouped(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw),
                               torch.from_numpy(offs).cuda(), scale_fmt="ue8m0")
    for g in range(len(counts)):
        lo, hi = int(offs[g]), int(offs[g + 1])
        rows = lo + sample_rows(hi - lo, 2, seed=g)
        y_ref, bnd = oracle.gemm(qa[rows], sa[rows], qw[g], sw[g])
        assert_gemm_close(y[torch.from_numpy(rows).cuda()], y_ref, bnd, "ue8m0 expert %d" % g)


@pytest.mark.parametrize("M", [128, 8])
def test_gemm_ue8m0_reports_non_power_of_two_scales(M):
    """M = 128 runs the block-scaled MMA, decode-sized M = 8 the promotion
    kernel; both check the scales' form (an activation scale, then a weight
    scale, no longer a power of two)."""
    x, qa, sa, qw, sw = _case(M, 256, 256, seed=7)
    bad_a = sa.copy()
    bad_a[5, 1] *= np.float32(1.5)                   # no longer a power of two
    fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(bad_a), cuda_codes(qw), cuda_f32(sw), scale_fmt="ue8m0")
    assert fp8bs.device_error() == fp8bs.ERR_SCALE
    assert fp8bs.device_error() == 0                 # read-and-clear
    bad_w = sw.copy()
    bad_w[1, 0] = np.float32(3e-3)
    fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(bad_w), scale_fmt="ue8m0")
    assert fp8bs.device_error() == fp8bs.ERR_SCALE
    # power-of-two scales raise nothing on either path
    fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw), scale_fmt="ue8m0")
    assert fp8bs.device_error() == 0
