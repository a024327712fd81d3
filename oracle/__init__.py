"""CPU oracle for the FP8 block-scaled linear path (TEST INFRASTRUCTURE ONLY).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.  Every function wraps the plain C in ``oracle.c``,
whose header cites the pages each step follows.

Arrays are numpy arrays (C-contiguous); bf16 data travels as ``uint16`` bit
patterns and e4m3fn codes as ``uint8``.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
values fixed by the pages, the format definitions, exact rational arithmetic
or an independent library routine.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        c_i64, c_int, c_p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode_array.restype = None
        lib.oracle_e4m3_encode_array.argtypes = [c_p, c_i64, c_p]
        lib.oracle_bf16_from_f32.restype = ctypes.c_uint16
        lib.oracle_bf16_from_f32.argtypes = [ctypes.c_float]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_ue8m0_round_up.restype = ctypes.c_float
        lib.oracle_ue8m0_round_up.argtypes = [ctypes.c_float]
        lib.oracle_block_scale.restype = ctypes.c_float
        lib.oracle_block_scale.argtypes = [ctypes.c_float, c_int]
        lib.oracle_act_quant.restype = None
        lib.oracle_act_quant.argtypes = [c_p, c_int, c_i64, c_i64, c_i64, c_int, c_p, c_p]
        lib.oracle_weight_quant.restype = None
        lib.oracle_weight_quant.argtypes = [c_p, c_i64, c_i64, c_i64, c_int, c_p, c_p]
        lib.oracle_weight_dequant.restype = None
        lib.oracle_weight_dequant.argtypes = [c_p, c_p, c_i64, c_i64, c_i64, c_int, c_p]
        lib.oracle_gemm.restype = None
        lib.oracle_gemm.argtypes = [c_p, c_p, c_p, c_p, c_i64, c_i64, c_i64, c_i64, c_i64, c_p, c_p]
        lib.oracle_act_quant_static.restype = None
        lib.oracle_act_quant_static.argtypes = [c_p, c_int, c_i64, c_i64, c_i64, c_p, c_i64, c_p]
        lib.oracle_act_dequant.restype = None
        lib.oracle_act_dequant.argtypes = [c_p, c_p, c_i64, c_i64, c_i64, c_i64, c_int, c_p]
        lib.oracle_num_threads.restype = c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError("expected %s, got %s" % (dtype, a.dtype))
    return a


def num_threads():
    """Threads the oracle's parallel loops use (OpenMP)."""
    return _load().oracle_num_threads()


def e4m3_decode(code):
    return _load().oracle_e4m3_decode(int(code))


def e4m3_encode(f):
    return _load().oracle_e4m3_encode(float(np.float32(f)))


def e4m3_encode_array(f):
    """Element-wise encode of an fp32 array (a loop over the scalar codec)."""
    f = np.ascontiguousarray(f, dtype=np.float32).ravel()
    out = np.empty(f.size, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(f), f.size, _ptr(out))
    return out


def e4m3_table():
    """All 256 decoded values (float64; NaN codes give NaN)."""
    lib = _load()
    return np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)


def bf16_from_f32(f):
    return _load().oracle_bf16_from_f32(float(np.float32(f)))


def ue8m0_round_up(s):
    return _load().oracle_ue8m0_round_up(float(np.float32(s)))


def block_scale(amax, ue8m0):
    return _load().oracle_block_scale(float(np.float32(amax)), int(bool(ue8m0)))


def act_quant(x, block=128, scale_fmt=None):
    """x: [rows, cols] bf16 bit patterns (uint16) or float32 -> (q uint8, s float32)."""
    if scale_fmt not in (None, "ue8m0"):
        raise ValueError("scale_fmt must be None or 'ue8m0'")
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        is_bf16 = 1
    elif x.dtype == np.float32:
        is_bf16 = 0
    else:
        raise TypeError("x must be bf16 bits (uint16) or float32")
    if x.ndim != 2:
        x = x.reshape(-1, x.shape[-1])
    rows, cols = x.shape
    if cols % block != 0:
        raise ValueError("last dimension must be a multiple of block")
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty((rows, cols // block), dtype=np.float32)
    _load().oracle_act_quant(_ptr(x), is_bf16, rows, cols, block,
                             int(scale_fmt == "ue8m0"), _ptr(q), _ptr(s))
    return q, s


def _act_input(x):
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, 1
    if x.dtype == np.float32:
        return x, 0
    raise TypeError("x must be bf16 bits (uint16) or float32")


def _scale_table(s, rows, nblk):
    """A static scale vector [nblk] (row stride 0) or a per-row table [rows, nblk]."""
    s = _c(s, np.float32)
    if s.shape == (nblk,):
        return s, 0
    if s.shape == (rows, nblk):
        return s, nblk
    raise ValueError("scales must be [cols/block] or [rows, cols/block]")


def act_quant_static(x, s, block=128):
    """Static activation scheme: q = e4m3(x / s) with precomputed scales.

    x: [rows, cols] bf16 bits (uint16) or float32; s: float32 [cols/block]
    (one scale per block of channels, shared by all rows) or [rows, cols/block].
    Returns q uint8 [rows, cols]."""
    x, is_bf16 = _act_input(x)
    rows, cols = x.shape
    if cols % block != 0:
        raise ValueError("last dimension must be a multiple of block")
    s, stride = _scale_table(s, rows, cols // block)
    q = np.empty((rows, cols), dtype=np.uint8)
    _load().oracle_act_quant_static(_ptr(x), is_bf16, rows, cols, block, _ptr(s), stride, _ptr(q))
    return q


def act_dequant(q, s, block=128, out="bf16"):
    """static_dequant: y = fp8 value * its block's scale (fp32 product).

    q: [rows, cols] uint8; s as for act_quant_static.  out="bf16" returns
    uint16 bit patterns, out="f32" float32."""
    q = _c(q, np.uint8)
    rows, cols = q.shape
    if cols % block != 0:
        raise ValueError("last dimension must be a multiple of block")
    s, stride = _scale_table(s, rows, cols // block)
    y = np.empty((rows, cols), dtype=np.uint16 if out == "bf16" else np.float32)
    _load().oracle_act_dequant(_ptr(q), _ptr(s), stride, rows, cols, block, int(out == "bf16"),
                               _ptr(y))
    return y


def weight_quant(w, block=128, scale_fmt=None):
    """w: [rows, cols] float32 -> (q uint8 [rows, cols], s float32 [cdiv, cdiv])."""
    w = _c(w, np.float32)
    rows, cols = w.shape
    rb, cb = -(-rows // block), -(-cols // block)
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty((rb, cb), dtype=np.float32)
    _load().oracle_weight_quant(_ptr(w), rows, cols, block,
                                int(scale_fmt == "ue8m0"), _ptr(q), _ptr(s))
    return q, s


def weight_dequant(q, s, block=128, out="bf16"):
    """q: [M, N] uint8, s: [cdiv(M,block), cdiv(N,block)] float32 -> y.

    out="bf16" returns uint16 bit patterns, out="f32" returns float32."""
    q = _c(q, np.uint8)
    s = _c(s, np.float32)
    M, N = q.shape
    if s.shape != (-(-M // block), -(-N // block)):
        raise ValueError("scale shape must be (cdiv(M,block), cdiv(N,block))")
    y = np.empty((M, N), dtype=np.uint16 if out == "bf16" else np.float32)
    _load().oracle_weight_dequant(_ptr(q), _ptr(s), M, N, block,
                                  int(out == "bf16"), _ptr(y))
    return y


def gemm(qa, sa, qw, sw, block=128, with_bound=True, w_scales="block"):
    """FP64 reference of y = A W^T on block-scaled FP8 operands.

    qa [M,K] uint8, sa [M,K/block] f32, qw [N,K] uint8, and sw
    [cdiv(N,block),K/block] f32 (w_scales="block": 128x128 weight blocks) or
    [N,K/block] (w_scales="row": one scale per row and K block, as for a
    second activation-like operand).
    Returns (y [M,N] float64, bound [M,N] float64 or None)."""
    qa = _c(qa, np.uint8)
    qw = _c(qw, np.uint8)
    sa = _c(sa, np.float32)
    sw = _c(sw, np.float32)
    M, K = qa.shape
    N = qw.shape[0]
    if qw.shape[1] != K or K % block:
        raise ValueError("bad K")
    if w_scales not in ("block", "row"):
        raise ValueError("w_scales must be 'block' or 'row'")
    sw_rows = block if w_scales == "block" else 1
    if sa.shape != (M, K // block) or sw.shape != (-(-N // sw_rows), K // block):
        raise ValueError("bad scale shapes")
    y = np.empty((M, N), dtype=np.float64)
    b = np.empty((M, N), dtype=np.float64) if with_bound else None
    _load().oracle_gemm(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), M, N, K, block, sw_rows,
                        _ptr(y), _ptr(b) if b is not None else None)
    return y, b


def act_quant_transposed(x, block=128, scale_fmt=None):
    """Quantization in block x 1 column blocks, written transposed: the
    operand layout of the weight-gradient GEMM, contracted over the rows of x.

    By definition this is act_quant of x^T: x [rows, cols] (bf16 bits or
    float32, rows % block == 0) -> q [cols, rows] uint8, s [cols, rows/block]."""
    x = np.ascontiguousarray(x)
    if x.ndim != 2:
        raise ValueError("x must be 2-D")
    return act_quant(np.ascontiguousarray(x.T), block, scale_fmt)


def fp8_transpose(q, s, block=128):
    """The transposed FP8 matrix with its transposed block scales (exact):
    q [R, C] uint8, s [cdiv(R,block), cdiv(C,block)] -> (q^T, s^T)."""
    q = _c(q, np.uint8)
    s = _c(s, np.float32)
    R, C = q.shape
    if s.shape != (-(-R // block), -(-C // block)):
        raise ValueError("scale shape must be (cdiv(R,block), cdiv(C,block))")
    return np.ascontiguousarray(q.T), np.ascontiguousarray(s.T)


def bf16_bits_to_f32(h):
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)
