"""The C-ABI library loads without a GPU, exports every entry point that
include/fp8bs.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import subprocess

import pytest

import fp8_block_scaled_10_b200 as fp8bs
from fp8_block_scaled_10_b200 import build as fbuild


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return fp8bs.lib()


def test_header_declares_the_boundary():
    names = fp8bs.header_symbols()
    for required in ("fp8bs_act_quant", "fp8bs_weight_dequant", "fp8bs_fp8_gemm",
                     "fp8bs_fp8_linear", "fp8bs_fp8_gemm_grouped", "fp8bs_weight_quant",
                     "fp8bs_gemm_workspace_size", "fp8bs_get_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fp8bs.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in fp8bs.header_symbols():
        assert name in exported, name
        assert getattr(L, name) is not None
    # nothing but the declared entry points is exported
    assert {n for n in exported if n.startswith("fp8bs_")} == set(fp8bs.header_symbols())


def test_status_strings(L):
    assert L.fp8bs_status_string(0) == b"FP8BS_OK"
    assert L.fp8bs_status_string(3) == b"FP8BS_ERR_WORKSPACE"
    assert L.fp8bs_version() >= 100


def _p(v):
    return ctypes.c_void_p(v)


def test_host_side_argument_errors_without_gpu(L):
    dummy = _p(4096)            # never dereferenced: validation fails first
    # K not a multiple of 128
    st = L.fp8bs_fp8_gemm(dummy, dummy, dummy, dummy, 8, 256, 100, dummy, None, 0, None)
    assert st == fp8bs.ERR_INVALID_ARG
    assert b"K=100" in L.fp8bs_last_error_message()
    # null operand
    st = L.fp8bs_fp8_gemm(None, dummy, dummy, dummy, 8, 256, 128, dummy, None, 0, None)
    assert st == fp8bs.ERR_INVALID_ARG
    # misaligned operand
    st = L.fp8bs_fp8_gemm(_p(4097), dummy, dummy, dummy, 8, 256, 128, dummy, None, 0, None)
    assert st == fp8bs.ERR_INVALID_ARG
    # block sizes other than 32, 64, 128 and 256 are not implemented
    st = L.fp8bs_act_quant(dummy, 0, 4, 192, 48, 0, dummy, dummy, None)
    assert st == fp8bs.ERR_UNSUPPORTED
    assert L.fp8bs_weight_dequant(dummy, dummy, 4, 4, 512, dummy, 0, None) == fp8bs.ERR_UNSUPPORTED
    assert L.fp8bs_weight_quant(dummy, 0, 4, 4, 16, 0, dummy, dummy, None) == fp8bs.ERR_UNSUPPORTED
    # last dimension not a multiple of the block
    st = L.fp8bs_act_quant(dummy, 0, 4, 200, 128, 0, dummy, dummy, None)
    assert st == fp8bs.ERR_INVALID_ARG
    # unknown scale format / dtype
    assert L.fp8bs_act_quant(dummy, 0, 4, 256, 128, 7, dummy, dummy, None) == fp8bs.ERR_INVALID_ARG
    assert L.fp8bs_weight_dequant(dummy, dummy, 4, 4, 128, dummy, 9, None) == fp8bs.ERR_INVALID_ARG
    # grouped: G out of range
    st = L.fp8bs_fp8_gemm_grouped(0, dummy, 8, dummy, dummy, dummy, dummy, 256, 128, dummy, None)
    assert st == fp8bs.ERR_INVALID_ARG
    # FP8-output GEMM: N must be a multiple of 128, the output format known
    st = L.fp8bs_fp8_gemm_quant(dummy, dummy, dummy, dummy, 8, 200, 128, 0, dummy, dummy, None, None)
    assert st == fp8bs.ERR_INVALID_ARG and b"N=200" in L.fp8bs_last_error_message()
    st = L.fp8bs_fp8_gemm_quant(dummy, dummy, dummy, dummy, 8, 256, 128, 5, dummy, dummy, None, None)
    assert st == fp8bs.ERR_INVALID_ARG
    st = L.fp8bs_fp8_gemm_quant(dummy, dummy, dummy, dummy, 8, 256, 128, 0, dummy, None, None, None)
    assert st == fp8bs.ERR_INVALID_ARG
    # FP32-output GEMM: the scale format must be known, K a multiple of 128
    st = L.fp8bs_fp8_gemm_f32(dummy, dummy, dummy, dummy, 8, 256, 128, 3, dummy, None, 0, None)
    assert st == fp8bs.ERR_INVALID_ARG
    st = L.fp8bs_fp8_gemm_f32(dummy, dummy, dummy, dummy, 8, 256, 96, 0, dummy, None, 0, None)
    assert st == fp8bs.ERR_INVALID_ARG and b"K=96" in L.fp8bs_last_error_message()
    # static activation scheme: scale row stride 0 or >= cols / block
    st = L.fp8bs_act_quant_static(dummy, 0, 4, 256, 128, dummy, 1, dummy, None, None)
    assert st == fp8bs.ERR_INVALID_ARG and b"s_row_stride" in L.fp8bs_last_error_message()
    st = L.fp8bs_act_quant_static(dummy, 0, 4, 200, 128, dummy, 0, dummy, None, None)
    assert st == fp8bs.ERR_INVALID_ARG
    st = L.fp8bs_act_quant_static(dummy, 0, 4, 256, 48, dummy, 0, dummy, None, None)
    assert st == fp8bs.ERR_UNSUPPORTED
    st = L.fp8bs_act_quant_static(dummy, 0, 4, 256, 128, None, 0, dummy, None, None)
    assert st == fp8bs.ERR_INVALID_ARG
    st = L.fp8bs_act_quant_static(dummy, 0, 4, 256, 128, dummy, 0, dummy, _p(4098), None)
    assert st == fp8bs.ERR_INVALID_ARG
    assert L.fp8bs_act_dequant(dummy, dummy, 1, 4, 256, 128, dummy, 0, None) == fp8bs.ERR_INVALID_ARG
    assert L.fp8bs_act_dequant(dummy, dummy, 0, 4, 256, 128, dummy, 7, None) == fp8bs.ERR_INVALID_ARG
    assert L.fp8bs_act_dequant(dummy, dummy, 0, 4, 256, 512, dummy, 0, None) == fp8bs.ERR_UNSUPPORTED
    # a tile count past the kernels' 32-bit unit indices is refused
    st = L.fp8bs_fp8_gemm(dummy, dummy, dummy, dummy, 1 << 31, 1 << 30, 128, dummy, None, 0, None)
    assert st == fp8bs.ERR_INVALID_ARG and b"too large" in L.fp8bs_last_error_message()
    # empty problems are successful no-ops
    assert L.fp8bs_act_quant_static(None, 0, 0, 256, 128, None, 0, None, None, None) == fp8bs.OK
    assert L.fp8bs_act_dequant(None, None, 2, 0, 256, 128, None, 0, None) == fp8bs.OK
    assert L.fp8bs_act_quant(None, 0, 0, 256, 128, 0, None, None, None) == fp8bs.OK
    assert L.fp8bs_weight_dequant(None, None, 0, 16, 128, None, 0, None) == fp8bs.OK
    assert L.fp8bs_fp8_gemm(dummy, dummy, dummy, dummy, 0, 256, 128, dummy, None, 0, None) == fp8bs.OK
    assert L.fp8bs_fp8_gemm_f32(dummy, dummy, dummy, dummy, 0, 256, 128, 1, dummy, None, 0,
                                None) == fp8bs.OK
    assert L.fp8bs_fp8_gemm_quant(dummy, dummy, dummy, dummy, 0, 256, 128, 0, dummy, dummy, None,
                                  None) == fp8bs.OK


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        fp8bs.act_quant(torch.zeros(4, 128, dtype=torch.bfloat16))


def test_every_entry_point_treats_an_empty_problem_as_a_no_op(L):
    """Zero rows (or an empty matrix) return OK before any device work, so
    these calls succeed on a host without a GPU."""
    dummy = _p(4096)
    OK = fp8bs.OK
    assert L.fp8bs_weight_quant(None, 0, 0, 256, 128, 0, None, None, None) == OK
    assert L.fp8bs_fp8_transpose(None, None, 0, 256, 128, None, None, None) == OK
    assert L.fp8bs_fp8_transpose(None, None, 256, 0, 128, None, None, None) == OK
    assert L.fp8bs_act_quant_transposed(None, 0, 0, 256, 128, 0, None, None, None) == OK
    assert L.fp8bs_fp8_gemm_ue8m0(dummy, dummy, dummy, dummy, 0, 256, 128, dummy, None, 0,
                                  None) == OK
    assert L.fp8bs_fp8_gemm_static_scratch(dummy, dummy, dummy, dummy, 0, 256, 128, dummy,
                                           None) == OK
    for fmt in (0, 1):
        assert L.fp8bs_fp8_gemm_rowwise(dummy, dummy, dummy, dummy, 0, 256, 128, fmt, dummy, 1,
                                        None, 0, None) == OK
    assert L.fp8bs_fp8_linear(None, 0, 256, 0, dummy, dummy, 128, dummy, dummy, dummy, None, 0,
                              None) == OK
    assert L.fp8bs_fp8_linear_ue8m0(None, 0, 256, dummy, dummy, 128, dummy, dummy, dummy, None, 0,
                                    None) == OK
    for fn in (L.fp8bs_fp8_gemm_grouped, L.fp8bs_fp8_gemm_grouped_ue8m0):
        assert fn(4, dummy, 0, dummy, dummy, dummy, dummy, 256, 128, dummy, None) == OK


def test_plain_c_client_builds_and_runs(L, tmp_path):
    """The header compiles as strict C99 and a C program links against the
    library and gets the documented host-side results (no Python involved)."""
    import os
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    libdir = os.path.dirname(fp8bs.LIB_PATH)
    exe = str(tmp_path / "abi_c_client")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(root, "include"), os.path.join(here, "abi_c_client.c"),
                    "-L", libdir, "-lfp8bs", "-Wl,-rpath," + libdir, "-o", exe],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "abi c client ok"


def _header_prototypes():
    """name -> list of parameter declarations, from include/fp8bs.h."""
    import os
    import re
    text = open(fp8bs.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    protos = {}
    for m in re.finditer(r"FP8BS_API\s+[^;(]*?\b(fp8bs_\w+)\s*\(([^)]*)\)\s*;", text, re.S):
        params = [p.strip() for p in m.group(2).split(",")]
        protos[m.group(1)] = [] if params == ["void"] else params
    return protos


def test_binding_signatures_match_the_header(L):
    """Every prototype's parameter count, and which parameters are pointers,
    agree with the ctypes argument types the binding declares."""
    import ctypes
    protos = _header_prototypes()
    assert set(protos) == set(fp8bs.header_symbols())
    for name, params in protos.items():
        fn = getattr(L, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == len(params), (name, params)
        for decl, ct in zip(params, fn.argtypes):
            is_ptr = "*" in decl
            assert is_ptr == (ct in (ctypes.c_void_p, ctypes.c_char_p) or
                              hasattr(ct, "contents") or
                              getattr(ct, "__name__", "").startswith("LP_")), (name, decl, ct)
            if is_ptr:
                continue
            # integer widths: int64_t, size_t, and int or an enum (C int)
            if "int64_t" in decl:
                want = ctypes.c_int64
            elif "size_t" in decl:
                want = ctypes.c_size_t
            else:
                assert decl.split()[0] in ("int", "fp8bs_dtype", "fp8bs_scale_fmt",
                                           "fp8bs_status"), (name, decl)
                want = ctypes.c_int
            assert ctypes.sizeof(ct) == ctypes.sizeof(want), (name, decl, ct)


def test_missing_library_fails_loudly(tmp_path):
    """Without the built library the binding raises instead of falling back."""
    code = ("import fp8_block_scaled_10_b200 as f\n"
            "f.LIB_PATH = %r\n"
            "f._lib = None\n"
            "try:\n"
            "    f.lib()\n"
            "except ImportError as e:\n"
            "    print('raised', e)\n" % str(tmp_path / "absent.so"))
    import os
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=root,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("raised"), r.stdout + r.stderr
