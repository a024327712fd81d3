"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Quantization and dequantization are compared byte for byte; the GEMM is held
to |dy| <= 4e-3 |y_ref| + 1e-3 sum_k |a_k w_k| against the oracle's FP64
result on the same dequantized operands.  Small cases span several tiles and
ragged tails; the full-size cases use the workload shapes the benchmark runs
(compared in full where the oracle is fast enough, else on sampled rows that
include every tile edge near both ends).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import workloads as wl

from _util import (assert_gemm_close, cuda_codes, cuda_f32, f32bits, quantized_weight,
                   sample_rows, u8)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_block_scaled_10_b200 import build
    build.build()
    torch.cuda.init()
    yield
    assert fp8bs.device_error() == 0


# --------------------------------------------------------------------------
# act_quant
# --------------------------------------------------------------------------

def _special_blocks(dtype):
    """Blocks that stress the scale rule and the e4m3 rounding:
    zeros, signed zeros, an exact-448 block with ties, tiny values, a single
    outlier, values that land exactly on e4m3 midpoints after the division."""
    rows = []
    z = np.zeros(128, np.float32)
    rows.append(z.copy())
    nz = z.copy(); nz[::2] = -0.0; rows.append(nz)
    t = np.array([448.0] + [1.0625, 1.1875, -3.25, 0.0009765625, -0.0029296875, 464.0 / 2,
                            2.0 ** -10, 3 * 2.0 ** -10] * 15 + [1.0] * 7, np.float32)[:128]
    rows.append(t)
    tiny = np.full(128, 1e-30, np.float32); tiny[5] = -3e-38; rows.append(tiny)
    out = np.random.default_rng(0).normal(0, 1, 128).astype(np.float32); out[17] = 5000.0
    rows.append(out)
    # x = m * s for e4m3 midpoints m, so fl32(x/s) sits on or next to a tie
    rng = np.random.default_rng(1)
    for a in (1.0, 3.0, 37.5, 0.1, 7e-3):
        s = np.float32(a) / np.float32(448.0)
        e = rng.integers(-6, 8, 128)
        k = rng.integers(0, 8, 128)
        m = ((8 + k) + 0.5) * np.exp2(e - 3.0)
        m = np.minimum(m, 440.0).astype(np.float32) * np.where(rng.random(128) < .5, -1, 1)
        x = (m * s).astype(np.float32)
        x[0] = np.float32(a)
        rows.append(x)
    x = np.stack(rows).astype(np.float32)
    if dtype == torch.bfloat16:
        return torch.from_numpy(x).to(torch.bfloat16)
    return torch.from_numpy(x)


def _oracle_act_quant(x_cpu, fmt):
    if x_cpu.dtype == torch.bfloat16:
        arr = wl.bf16_bits(x_cpu)
    else:
        arr = x_cpu.numpy()
    return oracle.act_quant(arr.reshape(-1, arr.shape[-1]), scale_fmt=fmt)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("fmt", [None, "ue8m0"])
@pytest.mark.parametrize("shape", [(1, 128), (3, 256), (129, 512), (1000, 1024), (2, 7, 384)])
def test_act_quant_bit_exact(shape, fmt, dtype):
    x = wl.normal_with_outliers(int(np.prod(shape[:-1])), shape[-1], seed=sum(shape),
                                frac=0.01, factor=50.0, dtype=dtype).reshape(shape)
    q, s = fp8bs.act_quant(x.cuda(), 128, fmt)
    assert q.dtype == torch.float8_e4m3fn and tuple(s.shape) == shape[:-1] + (shape[-1] // 128,)
    q_ref, s_ref = _oracle_act_quant(x, fmt)
    assert np.array_equal(u8(q).reshape(q_ref.shape), q_ref)
    assert np.array_equal(f32bits(s.cpu().numpy()).reshape(s_ref.shape), f32bits(s_ref))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("fmt", [None, "ue8m0"])
def test_act_quant_special_blocks(fmt, dtype):
    x = _special_blocks(dtype)
    q, s = fp8bs.act_quant(x.cuda(), 128, fmt)
    q_ref, s_ref = _oracle_act_quant(x, fmt)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))
    assert np.array_equal(u8(q), q_ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("fmt", [None, "ue8m0"])
def test_act_quant_infinite_blocks(fmt, dtype):
    """A block holding one +-inf: s = inf, every finite element of the block
    is the IEEE quotient x / inf = +-0 (codes 0x00 / 0x80), and the infinite
    element itself is inf / inf = NaN, whose sign IEEE leaves open (either
    NaN code is accepted there).  The other blocks are unaffected."""
    rows, cols = 64, 1024
    x = wl.normal_with_outliers(rows, cols, seed=91, frac=0.01, factor=50.0).float().numpy()
    rng = np.random.default_rng(92)
    inf_at = []
    for r in range(rows):
        for b in rng.choice(cols // 128, size=2, replace=False):
            c = int(b) * 128 + int(rng.integers(0, 128))
            x[r, c] = np.inf if rng.random() < 0.5 else -np.inf
            inf_at.append((r, c))
    xt = torch.from_numpy(x).to(dtype)
    q, s = fp8bs.act_quant(xt.cuda(), 128, fmt)
    q_ref, s_ref = _oracle_act_quant(xt, fmt)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))
    assert np.isinf(s_ref).sum() == len(inf_at)
    got = u8(q)
    nan_mask = np.zeros_like(got, dtype=bool)
    for r, c in inf_at:
        nan_mask[r, c] = True
    assert np.all((got[nan_mask] & 0x7F) == 0x7F) and np.all((q_ref[nan_mask] & 0x7F) == 0x7F)
    assert np.array_equal(got[~nan_mask], q_ref[~nan_mask])
    # every finite element of an infinite block encodes a signed zero
    blk_inf = np.repeat(np.isinf(s_ref), 128, axis=1) & ~nan_mask
    assert np.all((got[blk_inf] & 0x7F) == 0)


def test_act_quant_many_midpoints_fp32():
    """fp32 inputs built as e4m3 midpoint * s: the exact-division fallback runs often."""
    rng = np.random.default_rng(7)
    rows, cols = 512, 1024
    a = np.exp2(rng.uniform(-12, 8, (rows, cols // 128))).astype(np.float32)
    s = (a / np.float32(448.0)).astype(np.float32)
    e = rng.integers(-9, 8, (rows, cols))
    k = rng.integers(0, 16, (rows, cols))
    m = (k + 0.5) * np.exp2(e - 3.0)
    m = np.minimum(m, 440.0) * np.where(rng.random((rows, cols)) < .5, -1, 1)
    x = (m.astype(np.float32) * np.repeat(s, 128, axis=1)).astype(np.float32)
    x[:, ::128] = a
    xt = torch.from_numpy(x)
    q, sg = fp8bs.act_quant(xt.cuda())
    q_ref, s_ref = oracle.act_quant(x)
    assert np.array_equal(f32bits(sg.cpu().numpy()), f32bits(s_ref))
    assert np.array_equal(u8(q), q_ref)


@pytest.mark.parametrize("block", [32, 64, 256])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("fmt", [None, "ue8m0"])
def test_act_quant_other_block_sizes(block, fmt, dtype):
    """The configurable block_size: 1 x block scales, bit-exact with the oracle."""
    rows, cols = 257, 7 * 256
    x = wl.normal_with_outliers(rows, cols, seed=block + 3, frac=0.01, factor=50.0, dtype=dtype)
    q, s = fp8bs.act_quant(x.cuda(), block, fmt)
    arr = wl.bf16_bits(x) if dtype == torch.bfloat16 else x.numpy()
    q_ref, s_ref = oracle.act_quant(arr, block=block, scale_fmt=fmt)
    assert tuple(s.shape) == (rows, cols // block)
    assert np.array_equal(u8(q), q_ref)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))


@pytest.mark.parametrize("fmt", [None, "ue8m0"])
def test_act_quant_full_size(fmt):
    """act_quant on x bf16 [16384, 7168] ~N(0,1) with 0.1% entries x100, every byte."""
    x = wl.normal_with_outliers(16384, 7168, seed=20, frac=0.001, factor=100.0)
    q, s = fp8bs.act_quant(x.cuda(), 128, fmt)
    q_ref, s_ref = oracle.act_quant(wl.bf16_bits(x), scale_fmt=fmt)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))
    assert np.array_equal(u8(q), q_ref)


# --------------------------------------------------------------------------
# weight_dequant / weight_quant
# --------------------------------------------------------------------------

def _codes(M, N, seed):
    return wl.e4m3_codes(M, N, seed=seed).numpy()


@pytest.mark.parametrize("out", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(128, 128), (256, 576), (129, 130), (300, 1024), (1, 16), (5, 7)])
def test_weight_dequant_bit_exact(shape, out):
    M, N = shape
    q = _codes(M, N, seed=M + N)
    s = wl.uniform((-(-M // 128), -(-N // 128)), 1e-5, 1e-3, seed=3).numpy()
    s.flat[0] = -2.5e-4
    s.flat[-1] = 3.0e4
    y = fp8bs.weight_dequant(cuda_codes(q), cuda_f32(s), 128,
                             torch.bfloat16 if out == "bf16" else torch.float32)
    y_ref = oracle.weight_dequant(q, s, out=out)
    got = y.cpu().view(torch.int16).numpy().view(np.uint16) if out == "bf16" else y.cpu().numpy()
    if out == "f32":
        assert np.array_equal(f32bits(got), f32bits(y_ref))
    else:
        assert np.array_equal(got, y_ref)


@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_weight_dequant_every_code_and_scale_range(out):
    """All 256 codes (NaN codes 0x7F/0xFF included) against scales that span
    the kernel's two decode routes: |s| < 128 (shifted decode times s * 2^120),
    |s| >= 128 (integer decode), and a subnormal and a negative scale.
    Non-NaN outputs bit-exact; NaN exactly where the oracle has NaN."""
    M, N = 256, 1024
    q = (np.arange(M * N, dtype=np.int64) % 256).astype(np.uint8).reshape(M, N)
    q[1::2] = q[1::2, ::-1]
    s = np.array([[1.0, -3.5e-3, 127.99, 128.0, 3.0e30, 1e-40, 2.0 ** -20, 448.0],
                  [448.0, 2.0 ** -20, 1e-40, 3.0e30, 128.0, 127.99, -3.5e-3, 1.0]],
                 dtype=np.float32)
    y = fp8bs.weight_dequant(cuda_codes(q), cuda_f32(s), 128,
                             torch.bfloat16 if out == "bf16" else torch.float32)
    y_ref = oracle.weight_dequant(q, s, out=out)
    if out == "bf16":
        got = y.cpu().view(torch.int16).numpy().view(np.uint16)
        as_f = lambda b: (b.astype(np.uint32) << 16).view(np.float32)
        g, r = as_f(got), as_f(y_ref)
    else:
        got = y.cpu().numpy()
        g, r = got, y_ref
    assert np.array_equal(np.isnan(g), np.isnan(r))
    fin = ~np.isnan(r)
    assert fin.mean() > 0.99
    assert np.array_equal(f32bits(g[fin]), f32bits(r[fin]))


@pytest.mark.parametrize("block", [32, 64, 256])
@pytest.mark.parametrize("shape", [(300, 1024), (129, 130), (256, 7 * 64)])
def test_weight_dequant_other_block_sizes(block, shape):
    M, N = shape
    rng = np.random.default_rng(M + N + block)
    q = rng.integers(0, 254, (M, N)).astype(np.uint8)
    q = np.where(q >= 0x7F, q + 1, q).astype(np.uint8)
    s = rng.uniform(1e-5, 1e-3, (-(-M // block), -(-N // block))).astype(np.float32)
    y = fp8bs.weight_dequant(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), block)
    ref = oracle.weight_dequant(q, s, block=block)
    assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref)


@pytest.mark.parametrize("block", [32, 64, 256])
@pytest.mark.parametrize("fmt", [None, "ue8m0"])
def test_weight_quant_other_block_sizes(block, fmt):
    w = wl.weight_f32(300, 576, seed=block)
    q, s = fp8bs.weight_quant(w.cuda(), block, fmt)
    q_ref, s_ref = oracle.weight_quant(w.numpy(), block=block, scale_fmt=fmt)
    assert np.array_equal(u8(q), q_ref)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))


def test_weight_dequant_pages_example_shape():
    q = _codes(1024, 1024, seed=5)
    s = wl.uniform((8, 8), 1e-5, 1e-3, seed=6).numpy()
    y = fp8bs.weight_dequant(cuda_codes(q), cuda_f32(s))
    assert tuple(y.shape) == (1024, 1024)
    assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16),
                          oracle.weight_dequant(q, s))


def test_weight_dequant_full_size():
    """e4m3 W [18432, 7168] (all 254 finite codes), s [144, 56] ~U(1e-5, 1e-3) -> bf16."""
    q = _codes(18432, 7168, seed=30)
    s = wl.uniform((144, 56), 1e-5, 1e-3, seed=31).numpy()
    y = fp8bs.weight_dequant(cuda_codes(q), cuda_f32(s))
    assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16),
                          oracle.weight_dequant(q, s))


@pytest.mark.parametrize("fmt", [None, "ue8m0"])
@pytest.mark.parametrize("shape", [(256, 512), (300, 576), (129, 130), (128, 7168)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_weight_quant_bit_exact(shape, fmt, dtype):
    w = wl.weight_f32(*shape, seed=shape[0] * 7 + shape[1]).to(dtype)
    w[0, 0] = 0.5
    q, s = fp8bs.weight_quant(w.cuda(), 128, fmt)
    q_ref, s_ref = oracle.weight_quant(w.float().numpy(), scale_fmt=fmt)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(s_ref))
    assert np.array_equal(u8(q), q_ref)


# --------------------------------------------------------------------------
# fp8_gemm
# --------------------------------------------------------------------------

def _gemm_case(M, N, K, seed, fmt=None, heavy=False):
    if heavy:
        x = wl.heavy_tailed_channels(M, K, seed=seed)
    else:
        x = wl.normal_with_outliers(M, K, seed=seed, frac=0.01, factor=50.0)
    qa, sa = oracle.act_quant(wl.bf16_bits(x), scale_fmt=fmt)
    qw, sw = quantized_weight(N, K, seed=seed + 1, scale_fmt=fmt)
    return x, qa, sa, qw, sw


def test_gemm_tiny_linear():
    """x bf16 [128,512] ~N(0,1) with 1% entries x50; W [256,512]; y bf16 [128,256]."""
    x, qa, sa, qw, sw = _gemm_case(128, 256, 512, seed=0)
    assert sw.shape == (2, 4)
    y = fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw))
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "tiny")


@pytest.mark.parametrize("M,N,K", [
    (1, 256, 128), (127, 576, 512), (129, 130, 256), (300, 384, 1024), (256, 512, 7168),
    (513, 1280, 384), (64, 2048, 2048), (2, 18432, 256), (200, 136, 128),
    # 192-wide tiles whose columns straddle a 128-column weight block, a K
    # split of 192-wide tiles, and a last tile 64 columns wide
    (384, 200, 1024), (256, 576, 7168), (1000, 7168, 256),
])
def test_gemm_shapes(M, N, K):
    x, qa, sa, qw, sw = _gemm_case(M, N, K, seed=M + N + K)
    y = fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw))
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "gemm %dx%dx%d" % (M, N, K))


def test_gemm_split_tail_every_output():
    """160 tiles on 148 SMs: the 12 tiles of the last wave are split along K
    and summed by the tail reduction; ragged last row and column tiles."""
    M, N, K = 1200, 4000, 4096
    plan = fp8bs.gemm_plan(M, N, K)
    if fp8bs.lib().fp8bs_gemm_plan_string(M, N, K).decode().find("sms=148") < 0:
        pytest.skip("plan depends on the SM count: " + plan)
    assert "tail_splits=0" not in plan, plan
    x, qa, sa, qw, sw = _gemm_case(M, N, K, seed=77)
    y = fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw))
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "split tail " + plan)


def test_gemm_writes_only_its_output():
    """Canary rows and columns around y stay untouched (raw C-ABI call)."""
    M, N, K = 130, 200, 256
    x, qa, sa, qw, sw = _gemm_case(M, N, K, seed=99)
    a, a_s, w, w_s = cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw)
    big = torch.full((M + 2, N), -7.0, dtype=torch.bfloat16, device="cuda")
    y = big[1:M + 1]
    L = fp8bs.lib()
    st = L.fp8bs_fp8_gemm(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(a_s.data_ptr()),
                          ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(w_s.data_ptr()),
                          M, N, K, ctypes.c_void_p(y.data_ptr()), None, 0,
                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == fp8bs.OK
    torch.cuda.synchronize()
    assert torch.all(big[0] == -7.0) and torch.all(big[M + 1] == -7.0)
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "canary")


def test_gemm_is_deterministic():
    x, qa, sa, qw, sw = _gemm_case(64, 7168, 18432 // 4, seed=5, fmt="ue8m0")
    args = (cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw))
    y1 = fp8bs.fp8_gemm(*args)
    y2 = fp8bs.fp8_gemm(*args)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("K,N", wl.DECODE_KN)
@pytest.mark.parametrize("M", wl.DECODE_M)
def test_gemm_decode_full(M, K, N):
    """Decode shapes with ue8m0 scales, every output (split-K path where chosen)."""
    x, qa, sa, qw, sw = _gemm_case(M, N, K, seed=M * 3 + K, fmt="ue8m0")
    need = fp8bs.gemm_workspace_size(M, N, K)
    y = fp8bs.fp8_gemm(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw))
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "decode M=%d K=%d N=%d ws=%d" % (M, K, N, need))


@pytest.mark.parametrize("K,N", wl.PREFILL_KN)
def test_fp8_linear_prefill(K, N):
    """Fused act_quant + GEMM at M=4096 with heavy-tailed channels: q and s on every
    element, y on sampled rows (all columns)."""
    M = wl.PREFILL_M
    x = wl.heavy_tailed_channels(M, K, seed=40 + K)
    qw, sw = quantized_weight(N, K, seed=41 + N)
    y, q, s = fp8bs.fp8_linear(x.cuda(), cuda_codes(qw), cuda_f32(sw), return_quant=True)
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    assert np.array_equal(u8(q), qa)
    assert np.array_equal(f32bits(s.cpu().numpy()), f32bits(sa))
    rows = sample_rows(M, 12, seed=K + N)
    y_ref, bnd = oracle.gemm(qa[rows], sa[rows], qw, sw)
    assert_gemm_close(y[torch.from_numpy(rows).cuda()], y_ref, bnd, "prefill K=%d N=%d" % (K, N))


def test_fp8_linear_prefill_ue8m0_ragged():
    M, K, N = 1000, 7168, 576
    x = wl.heavy_tailed_channels(M, K, seed=50)
    qw, sw = quantized_weight(N, K, seed=51, scale_fmt="ue8m0")
    y = fp8bs.fp8_linear(x.cuda(), cuda_codes(qw), cuda_f32(sw), scale_fmt="ue8m0")
    qa, sa = oracle.act_quant(wl.bf16_bits(x), scale_fmt="ue8m0")
    y_ref, bnd = oracle.gemm(qa, sa, qw, sw)
    assert_gemm_close(y, y_ref, bnd, "ragged ue8m0")


# --------------------------------------------------------------------------
# grouped (expert-batched) GEMM
# --------------------------------------------------------------------------

def _grouped_case(counts, N, K, seed):
    G = len(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    Mt = int(offs[-1])
    x = wl.normal_with_outliers(max(Mt, 1), K, seed=seed, frac=0.001, factor=20.0)[:Mt]
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    qws, sws = zip(*[quantized_weight(N, K, seed=seed + 1 + g) for g in range(G)])
    return offs, qa, sa, np.stack(qws), np.stack(sws)


def test_grouped_small_ragged():
    counts = [0, 1, 130, 255, 64, 0, 300]
    N, K = 384, 256
    offs, qa, sa, qw, sw = _grouped_case(counts, N, K, seed=60)
    y = fp8bs.fp8_gemm_grouped(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw),
                               torch.from_numpy(offs).cuda())
    for g in range(len(counts)):
        lo, hi = offs[g], offs[g + 1]
        if hi == lo:
            continue
        y_ref, bnd = oracle.gemm(qa[lo:hi], sa[lo:hi], qw[g], sw[g])
        assert_gemm_close(y[lo:hi], y_ref, bnd, "group %d" % g)


def test_grouped_expert_config_sampled():
    """32 experts, W_e [2048, 7168], 65536 rows split ~Multinomial(65536, 1/32);
    every expert checked on rows at its tile edges plus random rows."""
    counts = wl.expert_counts(wl.EXPERT_TOKENS * wl.EXPERT_TOPK, wl.EXPERTS, seed=70).numpy()
    N, K = wl.EXPERT_FFN, wl.HIDDEN
    offs, qa, sa, qw, sw = _grouped_case(counts, N, K, seed=71)
    y = fp8bs.fp8_gemm_grouped(cuda_codes(qa), cuda_f32(sa), cuda_codes(qw), cuda_f32(sw),
                               torch.from_numpy(offs).cuda())
    for g in range(len(counts)):
        lo, hi = int(offs[g]), int(offs[g + 1])
        rows = lo + sample_rows(hi - lo, 2, seed=g)
        y_ref, bnd = oracle.gemm(qa[rows], sa[rows], qw[g], sw[g])
        assert_gemm_close(y[torch.from_numpy(rows).cuda()], y_ref, bnd, "expert %d" % g)


# --------------------------------------------------------------------------
# the division act_quant uses (scale_fmt None) against IEEE fp32 division
# --------------------------------------------------------------------------

def _adversarial_quotient_inputs(n, seed):
    rng = np.random.default_rng(seed)
    # x: bf16-like (8 significant bits), full fp32, near binade edges, tiny, zeros
    xb = rng.normal(0, 1, n).astype(np.float32)
    xb = (xb.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    xf = (rng.normal(0, 1, n) * np.exp2(rng.uniform(-40, 40, n))).astype(np.float32)
    edge = np.exp2(rng.integers(-30, 30, n)).astype(np.float32)
    edge = (edge.view(np.uint32) + rng.integers(-3, 4, n).astype(np.uint32)).view(np.float32)
    tiny = (rng.normal(0, 1, n) * 1e-38).astype(np.float32)
    x = np.concatenate([xb, xf, edge, tiny, np.float32([0.0, -0.0, 1.0, -1.0])])
    # s: a/448 for bf16 a (what act_quant divides by), random, all-ones significands, powers of 2
    a = np.abs(rng.normal(0, 10, len(x))).astype(np.float32) + np.float32(1e-4)
    a = (a.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    s1 = (a / np.float32(448.0)).astype(np.float32)
    s2 = np.exp2(rng.uniform(-22, 20, len(x))).astype(np.float32)
    s3 = ((rng.integers(100, 150, len(x)).astype(np.uint32) << 23) | np.uint32(0x7FFFFF)).view(np.float32)
    s4 = np.exp2(rng.integers(-22, 20, len(x)).astype(np.float32))
    pick = rng.integers(0, 4, len(x))
    s = np.choose(pick, [s1, s2, s3, s4]).astype(np.float32)
    return x, s


def test_quotient_matches_ieee_division():
    x, s = _adversarial_quotient_inputs(10_000_000, seed=90)
    ref = (x / s).astype(np.float32)            # numpy: IEEE fp32 division on the CPU
    xt, st = cuda_f32(x), cuda_f32(s)
    q = torch.empty_like(xt)
    L = fp8bs.lib()
    st_code = L.fp8bs_selftest_quotient(ctypes.c_void_p(xt.data_ptr()), ctypes.c_void_p(st.data_ptr()),
                                        ctypes.c_void_p(q.data_ptr()), x.size,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st_code == fp8bs.OK
    got = q.cpu().numpy()
    # Markstein's correction is exact while nothing underflows: compare the
    # fp32 quotient bitwise wherever numerator and quotient are >= 2^-100 ...
    big = (np.abs(x) >= np.float32(2.0 ** -100)) & (np.abs(ref) >= np.float32(2.0 ** -100))
    bad = big & (f32bits(got) != f32bits(ref))
    assert not bad.any(), (x[bad][:5], s[bad][:5], got[bad][:5], ref[bad][:5])
    assert big.mean() > 0.7
    # ... and everywhere, the e4m3 code act_quant derives from it
    assert np.array_equal(oracle.e4m3_encode_array(got), oracle.e4m3_encode_array(ref))


def _scale_selftest(amax, scale_fmt):
    s = torch.empty_like(amax)
    st_code = fp8bs.lib().fp8bs_selftest_block_scale(
        ctypes.c_void_p(amax.data_ptr()), ctypes.c_void_p(s.data_ptr()), amax.numel(),
        fp8bs.SCALE_FMT_UE8M0 if scale_fmt == "ue8m0" else fp8bs.SCALE_FMT_NONE,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st_code == fp8bs.OK
    return s


def test_block_scale_rule_every_float():
    """The kernels' scale max(amax, 1e-4) / 448 equals the correctly rounded
    fp32 quotient for every fp32 amax from 0 to +inf (checked against CUDA's
    IEEE division in torch, chunk by chunk), and ue8m0 rounds it up to a power
    of two; a sample is checked against the oracle's scale rule as well."""
    top = 0x7F800000                                   # +inf, included
    chunk = 1 << 27
    floor = torch.tensor(1e-4, dtype=torch.float32, device="cuda")
    for start in range(0, top + 1, chunk):
        bits = torch.arange(start, min(start + chunk, top + 1), dtype=torch.int32, device="cuda")
        amax = bits.view(torch.float32)
        # a tensor divisor: torch turns division by a Python scalar into a
        # multiplication by its reciprocal, which is not correctly rounded
        want = torch.maximum(amax, floor) / torch.full_like(amax, 448.0)
        got = _scale_selftest(amax, "none")
        bad = (got.view(torch.int32) != want.view(torch.int32))
        assert not bool(bad.any()), (amax[bad][:4].tolist(), got[bad][:4].tolist())
        up = _scale_selftest(amax, "ue8m0")
        m, e = torch.frexp(want)                        # want = m 2^e, m in [0.5, 1)
        want_up = torch.where((m == 0.5) | torch.isinf(want), want,
                              torch.ldexp(torch.ones_like(want), e))
        assert torch.equal(up.view(torch.int32), want_up.view(torch.int32))
        del bits, amax, want, got, up, m, e, want_up
    # zero, subnormals and values under the floor all give the floor's scale
    small = torch.tensor([0.0, 1e-45, 1e-38, 5e-5, 9.9999e-5], device="cuda")
    assert torch.equal(_scale_selftest(small, "none"),
                       torch.full_like(small, float(np.float32(1e-4) / np.float32(448))))
    # against the oracle on a sample spanning many binades
    rng = np.random.default_rng(5)
    sample = (10.0 ** rng.uniform(-6, 38, 4096)).astype(np.float32)
    sample[:3] = [np.float32(1e-4), np.float32(448.0), np.float32(np.inf)]
    for fmt in ("none", "ue8m0"):
        got = _scale_selftest(torch.from_numpy(sample).cuda(), fmt).cpu().numpy()
        ref = np.array([oracle.block_scale(float(a), fmt == "ue8m0") for a in sample],
                       dtype=np.float32)
        assert np.array_equal(f32bits(got), f32bits(ref)), fmt
