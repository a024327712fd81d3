"""Host-side argument checks of the Python binding (no GPU needed).

The C ABI takes raw pointers, so it cannot see a scale table that is too short
for its operand; the binding checks every shape before any device work.  On a
host without a GPU, a well-shaped call gets past those checks and stops at
the CUDA-tensor check, and a badly shaped one stops at its shape check."""
import pytest
import torch

import fp8_block_scaled_10_b200 as fp8bs


def _e4m3(*shape):
    return torch.zeros(*shape, dtype=torch.float8_e4m3fn)


def _f32(*shape):
    return torch.ones(*shape, dtype=torch.float32)


def _cuda_only(fn, *args, **kw):
    with pytest.raises(ValueError, match="CUDA tensors only"):
        fn(*args, **kw)


@pytest.mark.parametrize("lead,N,K", [((4,), 256, 512), ((2, 3), 130, 128), ((0,), 128, 256)])
def test_fp8_gemm_accepts_consistent_shapes(lead, N, K):
    a, a_s = _e4m3(*lead, K), _f32(*lead, K // 128)
    b, b_s = _e4m3(N, K), _f32(-(-N // 128), K // 128)
    _cuda_only(fp8bs.fp8_gemm, a, a_s, b, b_s)
    _cuda_only(fp8bs.fp8_gemm, a, a_s, b, b_s, scale_fmt="ue8m0", out_dtype=torch.float32)
    if N % 128 == 0:
        _cuda_only(fp8bs.fp8_gemm_quant, a, a_s, b, b_s)


@pytest.mark.parametrize("case,err,match", [
    ("a_s short", ValueError, "a_s must have shape"),
    ("a_s transposed", ValueError, "a_s must have shape"),
    ("b_s per row", ValueError, "b_s must have shape"),
    ("b_s bf16", TypeError, "b_s must be float32"),
    ("K mismatch", ValueError, "disagree on K"),
    ("K ragged", ValueError, "multiple of 128"),
    ("b 3-D", ValueError, "b must be 2-D"),
])
def test_fp8_gemm_rejects_inconsistent_shapes(case, err, match):
    M, N, K = 3, 256, 512
    a, a_s, b, b_s = _e4m3(M, K), _f32(M, K // 128), _e4m3(N, K), _f32(2, K // 128)
    if case == "a_s short":
        a_s = _f32(M - 1, K // 128)
    elif case == "a_s transposed":
        a_s = _f32(K // 128, M)
    elif case == "b_s per row":
        b_s = _f32(N, K // 128)
    elif case == "b_s bf16":
        b_s = b_s.to(torch.bfloat16)
    elif case == "K mismatch":
        b = _e4m3(N, K - 128)
    elif case == "K ragged":
        a, b = _e4m3(M, 200), _e4m3(N, 200)
    elif case == "b 3-D":
        b = _e4m3(1, N, K)
    with pytest.raises(err, match=match):
        fp8bs.fp8_gemm(a, a_s, b, b_s)


def test_fp8_gemm_quant_needs_whole_output_blocks():
    with pytest.raises(ValueError, match="multiple of 128 for an FP8 output"):
        fp8bs.fp8_gemm_quant(_e4m3(4, 256), _f32(4, 2), _e4m3(200, 256), _f32(2, 2))


def test_fp8_gemm_rowwise_shapes():
    M, N, K = 256, 384, 512
    _cuda_only(fp8bs.fp8_gemm_rowwise, _e4m3(M, K), _f32(M, 4), _e4m3(N, K), _f32(N, 4))
    with pytest.raises(ValueError, match="b_s must have shape"):
        fp8bs.fp8_gemm_rowwise(_e4m3(M, K), _f32(M, 4), _e4m3(N, K), _f32(3, 4))
    with pytest.raises(ValueError, match="expected"):
        fp8bs.fp8_gemm_rowwise(_e4m3(M, K), _f32(M, 4), _e4m3(N, K + 128), _f32(N, 5))


def test_fp8_linear_shapes():
    x = torch.zeros(3, 5, 256, dtype=torch.bfloat16)
    _cuda_only(fp8bs.fp8_linear, x, _e4m3(300, 256), _f32(3, 2))
    with pytest.raises(ValueError, match="weight_scale must have shape"):
        fp8bs.fp8_linear(x, _e4m3(300, 256), _f32(2, 2))
    with pytest.raises(ValueError, match="weight must be"):
        fp8bs.fp8_linear(x, _e4m3(300, 384), _f32(3, 3))
    with pytest.raises(TypeError, match="bfloat16"):
        fp8bs.fp8_linear(x.float(), _e4m3(300, 256), _f32(3, 2))


def test_fp8_linear_fused_shapes():
    x = torch.zeros(3, 5, 256, dtype=torch.bfloat16)
    _cuda_only(fp8bs.fp8_linear_fused, x, _e4m3(300, 256), _f32(3, 2))
    with pytest.raises(ValueError, match="weight_scale must have shape"):
        fp8bs.fp8_linear_fused(x, _e4m3(300, 256), _f32(2, 2))
    with pytest.raises(ValueError, match="weight must be"):
        fp8bs.fp8_linear_fused(x, _e4m3(300, 384), _f32(3, 3))
    with pytest.raises(TypeError, match="bfloat16"):
        fp8bs.fp8_linear_fused(x.float(), _e4m3(300, 256), _f32(3, 2))


def test_fp8_gemm_grouped_shapes():
    G, N, K, M = 4, 384, 256, 100
    offs = torch.tensor([0, 10, 10, 60, 100], dtype=torch.int64)
    good = (_e4m3(M, K), _f32(M, 2), _e4m3(G, N, K), _f32(G, 3, 2), offs)
    _cuda_only(fp8bs.fp8_gemm_grouped, *good)
    bad = list(good)
    bad[3] = _f32(G, 2, 2)
    with pytest.raises(ValueError, match="w_s must have shape"):
        fp8bs.fp8_gemm_grouped(*bad)
    bad = list(good)
    bad[4] = offs[:-1]
    with pytest.raises(ValueError, match="m_offsets must have shape"):
        fp8bs.fp8_gemm_grouped(*bad)
    bad = list(good)
    bad[4] = offs.int()
    with pytest.raises(TypeError, match="int64"):
        fp8bs.fp8_gemm_grouped(*bad)


def test_dtype_errors_are_type_errors():
    with pytest.raises(TypeError, match="out_dtype"):
        fp8bs._io_dtype(torch.float16, "out_dtype")


def test_operands_on_two_devices_are_refused():
    """Operands on different GPUs are refused before the kernel could take a
    peer pointer for a local one (checked with stand-in device objects)."""
    class Fake:
        is_cuda = True

        def __init__(self, dev):
            self.device = torch.device("cuda", dev)

        def is_contiguous(self):
            return True

    fp8bs._need_cuda(Fake(0), Fake(0))
    with pytest.raises(ValueError, match="one device"):
        fp8bs._need_cuda(Fake(0), Fake(1))
