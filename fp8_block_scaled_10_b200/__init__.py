"""FP8 block-scaled linear-layer kernels for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libfp8bs.so`` (``include/fp8bs.h``).
It only marshals arguments: tensors are allocated with torch on the current
CUDA device and every computation runs in the library's CUDA kernels on
torch's current stream.  There is no CPU fallback; if the library is missing
or cannot load, every call raises.

Calls keep the names and defaults of the DeepSeek-V3 inference kernels that
the pages describe:

* ``act_quant(x, block_size=128, scale_fmt=None) -> (q, s)``
* ``weight_dequant(x, s, block_size=128) -> y``
* ``fp8_gemm(a, a_s, b, b_s) -> y``
* ``fp8_linear(x, weight, weight_scale, scale_fmt=None) -> y``
* ``fp8_gemm_grouped(a, a_s, w, w_s, m_offsets) -> y``
* ``fp8_gemm_quant(a, a_s, b, b_s, out_scale_fmt=None) -> (q, s)`` (FP8 output)
* ``weight_quant(w, block_size=128, scale_fmt=None) -> (q, s)``
"""
import ctypes
import os
import re

import torch

__all__ = [
    "act_quant", "act_quant_static", "act_dequant", "static_dequant",
    "weight_dequant", "weight_quant", "fp8_gemm", "fp8_linear", "fp8_linear_fused",
    "fp8_gemm_grouped", "fp8_gemm_quant", "fp8_gemm_rowwise", "act_quant_transposed",
    "fp8_transpose", "gemm_workspace_size", "gemm_plan", "linear_plan", "device_error", "lib",
    "Fp8bsError",
    "LIB_PATH", "HEADER_PATH",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp8bs.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "fp8bs.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_SCALE = range(7)
DTYPE_BF16, DTYPE_F32 = 0, 1
SCALE_FMT_NONE, SCALE_FMT_UE8M0 = 0, 1


class Fp8bsError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s: %s" % (_STATUS_NAMES.get(status, status), message))
        self.status = status


_STATUS_NAMES = {OK: "FP8BS_OK", ERR_INVALID_ARG: "FP8BS_ERR_INVALID_ARG",
                 ERR_UNSUPPORTED: "FP8BS_ERR_UNSUPPORTED", ERR_WORKSPACE: "FP8BS_ERR_WORKSPACE",
                 ERR_CUDA: "FP8BS_ERR_CUDA", ERR_TIMEOUT: "FP8BS_ERR_TIMEOUT",
                 ERR_SCALE: "FP8BS_ERR_SCALE"}

_lib = None


def lib():
    """The loaded ``libfp8bs.so`` (ctypes.CDLL) with argument types declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libfp8bs.so is not built (python -m fp8_block_scaled_10_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sig = {
        "fp8bs_version": (i32, []),
        "fp8bs_status_string": (ctypes.c_char_p, [i32]),
        "fp8bs_last_error_message": (ctypes.c_char_p, []),
        "fp8bs_get_device_error": (i32, [p, ctypes.POINTER(i32)]),
        "fp8bs_act_quant": (i32, [p, i32, i64, i64, i64, i32, p, p, p]),
        "fp8bs_weight_dequant": (i32, [p, p, i64, i64, i64, p, i32, p]),
        "fp8bs_weight_quant": (i32, [p, i32, i64, i64, i64, i32, p, p, p]),
        "fp8bs_act_quant_static": (i32, [p, i32, i64, i64, i64, p, i64, p, p, p]),
        "fp8bs_act_quant_transposed": (i32, [p, i32, i64, i64, i64, i32, p, p, p]),
        "fp8bs_fp8_transpose": (i32, [p, p, i64, i64, i64, p, p, p]),
        "fp8bs_fp8_gemm_rowwise": (i32, [p, p, p, p, i64, i64, i64, i32, p, i32, p, sz, p]),
        "fp8bs_gemm_rowwise_workspace_size": (sz, [i64, i64, i64]),
        "fp8bs_act_dequant": (i32, [p, p, i64, i64, i64, i64, p, i32, p]),
        "fp8bs_gemm_workspace_size": (sz, [i64, i64, i64]),
        "fp8bs_gemm_plan_string": (ctypes.c_char_p, [i64, i64, i64]),
        "fp8bs_selftest_quotient": (i32, [p, p, p, i64, p]),
        "fp8bs_selftest_block_scale": (i32, [p, p, i64, i32, p]),
        "fp8bs_selftest_gemm_stall": (i32, [p, p, p, p, i64, i64, i64, p, p, sz, i32, p]),
        "fp8bs_fp8_gemm": (i32, [p, p, p, p, i64, i64, i64, p, p, sz, p]),
        "fp8bs_fp8_gemm_static_scratch": (i32, [p, p, p, p, i64, i64, i64, p, p]),
        "fp8bs_fp8_linear": (i32, [p, i64, i64, i32, p, p, i64, p, p, p, p, sz, p]),
        "fp8bs_linear_workspace_size": (sz, [i64, i64, i64]),
        "fp8bs_fp8_linear_fused": (i32, [p, i64, i64, i32, p, p, i64, p, p, p, p, sz, p]),
        "fp8bs_linear_plan_string": (ctypes.c_char_p, [i64, i64, i64]),
        "fp8bs_fp8_gemm_ue8m0": (i32, [p, p, p, p, i64, i64, i64, p, p, sz, p]),
        "fp8bs_fp8_gemm_f32": (i32, [p, p, p, p, i64, i64, i64, i32, p, p, sz, p]),
        "fp8bs_fp8_linear_ue8m0": (i32, [p, i64, i64, p, p, i64, p, p, p, p, sz, p]),
        "fp8bs_fp8_gemm_grouped_ue8m0": (i32, [i64, p, i64, p, p, p, p, i64, i64, p, p]),
        "fp8bs_fp8_gemm_grouped": (i32, [i64, p, i64, p, p, p, p, i64, i64, p, p]),
        "fp8bs_fp8_gemm_quant": (i32, [p, p, p, p, i64, i64, i64, i32, p, p, p, p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def header_symbols():
    """Names of the entry points that include/fp8bs.h declares."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"FP8BS_API[^;(]*?\b(fp8bs_\w+)\s*\(", text)))


def _check(status):
    if status != OK:
        msg = lib().fp8bs_last_error_message().decode(errors="replace")
        raise Fp8bsError(status, msg)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("fp8bs runs on CUDA tensors only (got a %s tensor)" % t.device)
        if not t.is_contiguous():
            raise ValueError("fp8bs expects contiguous tensors")
        if t.device != ts[0].device:
            raise ValueError("all operands must be on one device (%s and %s)"
                             % (ts[0].device, t.device))


def _codes(t):
    """uint8 view of an e4m3fn (or uint8) tensor."""
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8)
    if t.dtype == torch.uint8:
        return t
    raise TypeError("expected float8_e4m3fn or uint8 codes, got %s" % t.dtype)


def _scale_fmt(scale_fmt):
    if scale_fmt is None:
        return SCALE_FMT_NONE
    if scale_fmt == "ue8m0":
        return SCALE_FMT_UE8M0
    raise ValueError("scale_fmt must be None or 'ue8m0'")


def _io_dtype(dtype, what):
    """DTYPE_BF16 / DTYPE_F32 for a bfloat16 / float32 tensor dtype."""
    if dtype == torch.bfloat16:
        return DTYPE_BF16
    if dtype == torch.float32:
        return DTYPE_F32
    raise TypeError("%s must be torch.bfloat16 or torch.float32, got %s" % (what, dtype))


def _cdiv(a, b):
    return -(-a // b)


def _scales_like(s, shape, what):
    """Raise unless s is a float32 tensor of exactly ``shape``: the kernels read
    scales through raw pointers, so a short table would be read past its end."""
    if s.dtype != torch.float32:
        raise TypeError("%s must be float32, got %s" % (what, s.dtype))
    if tuple(s.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (what, tuple(shape), tuple(s.shape)))


def _gemm_operands(a, a_s, b, b_s):
    """Shape checks of fp8_gemm's operands -> (M, N, K)."""
    if b.dim() != 2:
        raise ValueError("b must be 2-D [N, K]")
    K = a.shape[-1]
    if b.shape[1] != K:
        raise ValueError("a [..., K] and b [N, K] disagree on K (%d vs %d)" % (K, b.shape[1]))
    if K <= 0 or K % 128 != 0:
        raise ValueError("K=%d must be a positive multiple of 128" % K)
    N = b.shape[0]
    _scales_like(a_s, tuple(a.shape[:-1]) + (K // 128,), "a_s")
    _scales_like(b_s, (_cdiv(N, 128), K // 128), "b_s")
    return a.numel() // K, N, K


def act_quant(x, block_size=128, scale_fmt=None):
    """Dynamic 1 x block_size quantization of the last dimension.

    Returns ``q`` (float8_e4m3fn, same shape as x) and ``s`` (float32,
    ``x.shape[:-1] + (x.shape[-1] // block_size,)``)."""
    _need_cuda(x)
    if x.dtype == torch.bfloat16:
        dt = DTYPE_BF16
    elif x.dtype == torch.float32:
        dt = DTYPE_F32
    else:
        raise TypeError("x must be bfloat16 or float32")
    if x.shape[-1] % block_size != 0:
        raise ValueError("last dimension must be a multiple of block_size")
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    s = torch.empty(*x.shape[:-1], cols // block_size, dtype=torch.float32, device=x.device)
    _check(lib().fp8bs_act_quant(_ptr(x), dt, rows, cols, block_size, _scale_fmt(scale_fmt),
                                 _ptr(q), _ptr(s), _stream(x.device)))
    return q, s


def _act_scales(s, lead, cols, block_size):
    """Row stride of a static scale vector [cols/block] (0) or a per-row table
    [..., cols/block] (cols/block)."""
    nblk = cols // block_size
    if s.dtype != torch.float32 or not s.is_contiguous():
        raise ValueError("scales must be contiguous float32")
    if tuple(s.shape) == (nblk,):
        return 0
    if tuple(s.shape) == tuple(lead) + (nblk,):
        return nblk
    raise ValueError("scales must be [cols/block] (static) or x.shape[:-1] + [cols/block]")


def act_quant_static(x, s, block_size=128, return_scales=False):
    """Static activation scheme: q = e4m3(x / s) with precomputed scales, no amax.

    s: float32 [cols/block_size] (one scale per block of channels, shared by
    every row) or a per-row table shaped like act_quant's.  Values beyond
    448 * s saturate.  With return_scales, also returns the per-row table
    ``x.shape[:-1] + (cols/block_size,)`` that fp8_gemm takes as a_s."""
    _need_cuda(x, s)
    if x.dtype == torch.bfloat16:
        dt = DTYPE_BF16
    elif x.dtype == torch.float32:
        dt = DTYPE_F32
    else:
        raise TypeError("x must be bfloat16 or float32")
    cols = x.shape[-1]
    if cols % block_size != 0:
        raise ValueError("last dimension must be a multiple of block_size")
    stride = _act_scales(s, x.shape[:-1], cols, block_size)
    rows = x.numel() // cols if cols else 0
    q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    s_out = torch.empty(*x.shape[:-1], cols // block_size, dtype=torch.float32,
                        device=x.device) if return_scales else None
    _check(lib().fp8bs_act_quant_static(_ptr(x), dt, rows, cols, block_size, _ptr(s), stride,
                                        _ptr(q), _ptr(s_out), _stream(x.device)))
    return (q, s_out) if return_scales else q


def act_dequant(q, s, block_size=128, out_dtype=torch.float32):
    """y = q.float() * s per 1 x block_size block (the pages' static_dequant).

    s as for act_quant_static (a static vector or act_quant's per-row
    table); the fp32 product is returned as float32 or rounded to bfloat16."""
    q = _codes(q)
    _need_cuda(q, s)
    cols = q.shape[-1]
    if cols % block_size != 0:
        raise ValueError("last dimension must be a multiple of block_size")
    stride = _act_scales(s, q.shape[:-1], cols, block_size)
    rows = q.numel() // cols if cols else 0
    dt = _io_dtype(out_dtype, "out_dtype")
    y = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    _check(lib().fp8bs_act_dequant(_ptr(q), _ptr(s), stride, rows, cols, block_size, _ptr(y), dt,
                                   _stream(q.device)))
    return y


static_dequant = act_dequant


def weight_dequant(x, s, block_size=128, out_dtype=torch.bfloat16):
    """y[i, j] = x[i, j] * s[i // block_size, j // block_size] (fp32 product,
    rounded to ``out_dtype``, bfloat16 or float32)."""
    x = _codes(x)
    _need_cuda(x, s)
    if x.dim() != 2:
        raise ValueError("weight_dequant expects a 2-D weight")
    M, N = x.shape
    if tuple(s.shape) != (-(-M // block_size), -(-N // block_size)) or s.dtype != torch.float32:
        raise ValueError("s must be float32 of shape (cdiv(M, block), cdiv(N, block))")
    dt = _io_dtype(out_dtype, "out_dtype")
    y = torch.empty(M, N, dtype=out_dtype, device=x.device)
    _check(lib().fp8bs_weight_dequant(_ptr(x), _ptr(s), M, N, block_size, _ptr(y), dt,
                                      _stream(x.device)))
    return y


def weight_quant(w, block_size=128, scale_fmt=None):
    """block_size x block_size quantization of a dense 2-D weight -> (q e4m3fn, s float32)."""
    _need_cuda(w)
    if w.dim() != 2:
        raise ValueError("weight_quant expects a 2-D weight")
    dt = _io_dtype(w.dtype, "w")
    M, N = w.shape
    q = torch.empty(M, N, dtype=torch.float8_e4m3fn, device=w.device)
    s = torch.empty(-(-M // block_size), -(-N // block_size), dtype=torch.float32, device=w.device)
    _check(lib().fp8bs_weight_quant(_ptr(w), dt, M, N, block_size, _scale_fmt(scale_fmt),
                                    _ptr(q), _ptr(s), _stream(w.device)))
    return q, s


def act_quant_transposed(x, block_size=128, scale_fmt=None):
    """Quantization in block_size x 1 column blocks, written transposed:
    act_quant(x.T) for a 2-D x [rows, cols] (rows % block_size == 0).

    Returns q [cols, rows] float8_e4m3fn and s [cols, rows // block_size]
    float32, the K-major operand of the weight-gradient GEMM."""
    _need_cuda(x)
    if x.dim() != 2:
        raise ValueError("act_quant_transposed expects a 2-D x")
    dt = _io_dtype(x.dtype, "x")
    rows, cols = x.shape
    q = torch.empty(cols, rows, dtype=torch.float8_e4m3fn, device=x.device)
    s = torch.empty(cols, rows // block_size, dtype=torch.float32, device=x.device)
    _check(lib().fp8bs_act_quant_transposed(_ptr(x), dt, rows, cols, block_size,
                                            _scale_fmt(scale_fmt), _ptr(q), _ptr(s),
                                            _stream(x.device)))
    return q, s


def fp8_transpose(q, s, block_size=128):
    """(q^T, s^T) of an FP8 matrix with block_size x block_size scales, exact."""
    q = _codes(q)
    _need_cuda(q, s)
    R, C = q.shape
    if tuple(s.shape) != (-(-R // block_size), -(-C // block_size)) or s.dtype != torch.float32:
        raise ValueError("s must be float32 of shape (cdiv(R, block), cdiv(C, block))")
    qt = torch.empty(C, R, dtype=torch.float8_e4m3fn, device=q.device)
    st = torch.empty(s.shape[1], s.shape[0], dtype=torch.float32, device=q.device)
    _check(lib().fp8bs_fp8_transpose(_ptr(q), _ptr(s.contiguous()), R, C, block_size,
                                     _ptr(qt), _ptr(st), _stream(q.device)))
    return qt, st


def fp8_gemm_rowwise(a, a_s, b, b_s, scale_fmt=None, out_dtype=torch.float32):
    """y = a @ b^T where both operands carry one scale per row and 128-wide
    K block (a_s [M, K/128], b_s [N, K/128]): the weight-gradient GEMM
    dW = dy^T x on act_quant_transposed(dy) and act_quant_transposed(x).
    out_dtype float32 (the default: weight gradients stay FP32) or bfloat16."""
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
    a, b = _codes(a), _codes(b)
    if a.dim() != 2 or b.dim() != 2 or b.shape[1] != a.shape[1]:
        raise ValueError("a [M,K], a_s [M,K/128], b [N,K], b_s [N,K/128] expected")
    M, K = a.shape
    N = b.shape[0]
    if K <= 0 or K % 128 != 0:
        raise ValueError("K=%d must be a positive multiple of 128" % K)
    _scales_like(a_s, (M, K // 128), "a_s")
    _scales_like(b_s, (N, K // 128), "b_s")
    _need_cuda(a, a_s, b, b_s)
    y = torch.empty(M, N, dtype=out_dtype, device=a.device)
    nws = int(lib().fp8bs_gemm_rowwise_workspace_size(M, N, K))
    ws = torch.empty(nws, dtype=torch.uint8, device=a.device) if nws else None
    dt = DTYPE_F32 if out_dtype == torch.float32 else DTYPE_BF16
    _check(lib().fp8bs_fp8_gemm_rowwise(_ptr(a), _ptr(a_s), _ptr(b), _ptr(b_s), M, N, K,
                                        _scale_fmt(scale_fmt), _ptr(y), dt, _ptr(ws), nws,
                                        _stream(a.device)))
    return y


def gemm_workspace_size(M, N, K):
    """Bytes of scratch fp8_gemm needs for an M x N x K problem on this device."""
    return int(lib().fp8bs_gemm_workspace_size(M, N, K))


def linear_plan(M, N, K):
    """Which form fp8_linear takes for this shape on the current device
    (fused act_quant + GEMM in one launch, or the two launches)."""
    return lib().fp8bs_linear_plan_string(M, N, K).decode()


def gemm_plan(M, N, K):
    """The launch plan fp8_gemm uses for an M x N x K problem on this device."""
    return lib().fp8bs_gemm_plan_string(M, N, K).decode()


def _workspace(M, N, K, device):
    n = gemm_workspace_size(M, N, K)
    if n == 0:
        return None, 0
    return torch.empty(n, dtype=torch.uint8, device=device), n


def fp8_gemm(a, a_s, b, b_s, scale_fmt=None, out_dtype=torch.bfloat16):
    """y = a @ b^T on block-scaled FP8 operands.

    a: [..., K] e4m3fn, a_s: [..., K/128] float32, b: [N, K] e4m3fn,
    b_s: [cdiv(N,128), K/128] float32 -> y: [..., N] of out_dtype
    (torch.bfloat16, or torch.float32 for the unrounded FP32 accumulator).
    scale_fmt="ue8m0" promises that every scale is a power of two: the tensor
    core's block-scaled MMA applies them (at decode-sized M, up to 64 rows, the
    promotion kernel runs instead, with a check of the scales)."""
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
    a, b = _codes(a), _codes(b)
    M, N, K = _gemm_operands(a, a_s, b, b_s)
    fmt = _scale_fmt(scale_fmt)
    _need_cuda(a, a_s, b, b_s)
    y = torch.empty(*a.shape[:-1], N, dtype=out_dtype, device=a.device)
    ws, nws = _workspace(M, N, K, a.device)
    if out_dtype == torch.float32:
        _check(lib().fp8bs_fp8_gemm_f32(_ptr(a), _ptr(a_s), _ptr(b), _ptr(b_s), M, N, K, fmt,
                                        _ptr(y), _ptr(ws), nws, _stream(a.device)))
        return y
    fn = lib().fp8bs_fp8_gemm_ue8m0 if fmt else lib().fp8bs_fp8_gemm
    _check(fn(_ptr(a), _ptr(a_s), _ptr(b), _ptr(b_s), M, N, K, _ptr(y), _ptr(ws), nws,
              _stream(a.device)))
    return y


def fp8_gemm_quant(a, a_s, b, b_s, out_scale_fmt=None, return_y=False):
    """fp8_gemm with an FP8 output: y = a @ b^T rounded to bf16, then quantized
    per 1x128 block of each row as act_quant(y, 128, out_scale_fmt) would.

    Returns (q e4m3fn [..., N], s float32 [..., N/128]), plus the bf16 y when
    return_y.  N must be a multiple of 128."""
    a, b = _codes(a), _codes(b)
    M, N, K = _gemm_operands(a, a_s, b, b_s)
    if N % 128 != 0:
        raise ValueError("N=%d must be a multiple of 128 for an FP8 output" % N)
    _need_cuda(a, a_s, b, b_s)
    q = torch.empty(*a.shape[:-1], N, dtype=torch.uint8, device=a.device)
    s = torch.empty(*a.shape[:-1], N // 128, dtype=torch.float32, device=a.device)
    y = torch.empty(*a.shape[:-1], N, dtype=torch.bfloat16, device=a.device) if return_y else None
    _check(lib().fp8bs_fp8_gemm_quant(_ptr(a), _ptr(a_s), _ptr(b), _ptr(b_s), M, N, K,
                                      _scale_fmt(out_scale_fmt), _ptr(q), _ptr(s), _ptr(y),
                                      _stream(a.device)))
    q = q.view(torch.float8_e4m3fn)
    return (q, s, y) if return_y else (q, s)


def fp8_linear(x, weight, weight_scale, scale_fmt=None, return_quant=False,
               weight_scale_fmt=None):
    """FP8 linear forward: act_quant(x) then fp8_gemm with the block-scaled weight.

    x: [..., K] bfloat16, weight: [N, K] e4m3fn, weight_scale: [cdiv(N,128), K/128].
    With scale_fmt="ue8m0" and weight_scale_fmt="ue8m0" (power-of-two weight
    scales) the GEMM is the ue8m0 entry (block-scaled MMA; promotion kernel at
    decode-sized M)."""
    w = _codes(weight)
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    if w.dim() != 2 or w.shape[1] != x.shape[-1]:
        raise ValueError("weight must be [N, K] with K = x.shape[-1]")
    K = x.shape[-1]
    if K <= 0 or K % 128 != 0:
        raise ValueError("K=%d must be a positive multiple of 128" % K)
    N = w.shape[0]
    _scales_like(weight_scale, (_cdiv(N, 128), K // 128), "weight_scale")
    _need_cuda(x, w, weight_scale)
    M = x.numel() // K
    y = torch.empty(*x.shape[:-1], N, dtype=torch.bfloat16, device=x.device)
    q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    s = torch.empty(*x.shape[:-1], K // 128, dtype=torch.float32, device=x.device)
    if _scale_fmt(scale_fmt) and _scale_fmt(weight_scale_fmt):
        ws, nws = _workspace(M, N, K, x.device)
        _check(lib().fp8bs_fp8_linear_ue8m0(_ptr(x), M, K, _ptr(w), _ptr(weight_scale), N,
                                            _ptr(y), _ptr(q), _ptr(s), _ptr(ws), nws,
                                            _stream(x.device)))
    else:
        nws = int(lib().fp8bs_linear_workspace_size(M, N, K))
        ws = torch.empty(nws, dtype=torch.uint8, device=x.device) if nws else None
        _check(lib().fp8bs_fp8_linear(_ptr(x), M, K, _scale_fmt(scale_fmt), _ptr(w),
                                      _ptr(weight_scale), N, _ptr(y), _ptr(q), _ptr(s), _ptr(ws),
                                      nws, _stream(x.device)))
    return (y, q, s) if return_quant else y


def fp8_linear_fused(x, weight, weight_scale, scale_fmt=None, return_quant=False):
    """The FP8 linear forward as one launch: the SMs the GEMM's tiles leave
    idle quantize x (act_quant, bit-identical q and s) while the GEMM
    consumes it.  Raises (FP8BS_ERR_UNSUPPORTED) where no such launch exists:
    decode-sized M, or tiles that fill the GPU.  fp8_linear picks this form
    itself when the planner expects it to be faster (linear_plan names the
    choice).  x: [..., K] bfloat16, weight: [N, K] e4m3fn, weight_scale:
    [cdiv(N,128), K/128]; scale_fmt sets the activation scales' format."""
    w = _codes(weight)
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    if w.dim() != 2 or w.shape[1] != x.shape[-1]:
        raise ValueError("weight must be [N, K] with K = x.shape[-1]")
    K = x.shape[-1]
    if K <= 0 or K % 128 != 0:
        raise ValueError("K=%d must be a positive multiple of 128" % K)
    N = w.shape[0]
    _scales_like(weight_scale, (_cdiv(N, 128), K // 128), "weight_scale")
    _need_cuda(x, w, weight_scale)
    M = x.numel() // K
    y = torch.empty(*x.shape[:-1], N, dtype=torch.bfloat16, device=x.device)
    q = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    s = torch.empty(*x.shape[:-1], K // 128, dtype=torch.float32, device=x.device)
    nws = int(lib().fp8bs_linear_workspace_size(M, N, K))
    ws = torch.empty(nws, dtype=torch.uint8, device=x.device) if nws else None
    _check(lib().fp8bs_fp8_linear_fused(_ptr(x), M, K, _scale_fmt(scale_fmt), _ptr(w),
                                        _ptr(weight_scale), N, _ptr(y), _ptr(q), _ptr(s),
                                        _ptr(ws), nws, _stream(x.device)))
    return (y, q, s) if return_quant else y


def fp8_gemm_grouped(a, a_s, w, w_s, m_offsets, scale_fmt=None):
    """Per-expert FP8 GEMMs over rows grouped contiguously by expert.

    a: [M_total, K] e4m3fn, a_s: [M_total, K/128], w: [G, N, K] e4m3fn,
    w_s: [G, cdiv(N,128), K/128], m_offsets: [G+1] int64 on the device."""
    a, w = _codes(a), _codes(w)
    if m_offsets.dtype != torch.int64:
        raise TypeError("m_offsets must be int64")
    if a.dim() != 2 or w.dim() != 3 or w.shape[2] != a.shape[1]:
        raise ValueError("a [M_total, K] and w [G, N, K] expected")
    G, N, K = w.shape
    M = a.shape[0]
    if K <= 0 or K % 128 != 0:
        raise ValueError("K=%d must be a positive multiple of 128" % K)
    if tuple(m_offsets.shape) != (G + 1,):
        raise ValueError("m_offsets must have shape (G + 1,) = (%d,)" % (G + 1))
    _scales_like(a_s, (M, K // 128), "a_s")
    _scales_like(w_s, (G, _cdiv(N, 128), K // 128), "w_s")
    _need_cuda(a, a_s, w, w_s, m_offsets)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=a.device)
    fn = lib().fp8bs_fp8_gemm_grouped_ue8m0 if _scale_fmt(scale_fmt) else lib().fp8bs_fp8_gemm_grouped
    _check(fn(G, _ptr(m_offsets), M, _ptr(a), _ptr(a_s), _ptr(w), _ptr(w_s), N, K, _ptr(y),
              _stream(a.device)))
    return y


def device_error(device=None):
    """Synchronize the current stream, then read and clear the device error word."""
    code = ctypes.c_int(0)
    _check(lib().fp8bs_get_device_error(_stream(device), ctypes.byref(code)))
    return code.value
