"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each test checks one oracle function against something it does not compute
itself: a constant or worked shape the pages state (tests/golden), the e4m3fn
and bf16 format definitions as implemented by torch's own casts (library
routines), exact rational or integer arithmetic, closed forms and invariants.
The cases are chosen so that a plausible slip (a dropped scale, a transposed
operand, a swapped scale index, a wrong constant, a floor instead of a ceiling
division) fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")
FACTS = json.load(open(GOLDEN))
E4M3_MAX = FACTS["e4m3_max"]["value"]
CLAMP = FACTS["amax_clamp_min"]["value"]
BLOCK = FACTS["block_size"]["value"]


def f32(v):
    return np.float32(v)


def torch_e4m3_bytes(a):
    """torch's own fp32 -> float8_e4m3fn cast, as raw bytes."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# --------------------------------------------------------------------------
# e4m3fn codec
# --------------------------------------------------------------------------

def test_e4m3_decode_table_matches_torch_dtype():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = oracle.e4m3_table()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    # signed zeros
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))


def test_e4m3_decode_format_facts():
    assert FACTS["e4m3_bits"]["exponent_bits"] == 4 and FACTS["e4m3_bits"]["mantissa_bits"] == 3
    assert oracle.e4m3_decode(0x7E) == E4M3_MAX          # largest finite value, 448
    assert oracle.e4m3_decode(0xFE) == -E4M3_MAX
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6          # smallest normal
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9          # smallest subnormal
    assert oracle.e4m3_decode(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert oracle.e4m3_decode(0x38) == 1.0                # exponent bias 7
    v = oracle.e4m3_decode(0x80)
    assert v == 0.0 and math.copysign(1.0, v) < 0
    finite = [oracle.e4m3_decode(c) for c in range(256) if c & 0x7F != 0x7F]
    assert max(finite) == E4M3_MAX and min(finite) == -E4M3_MAX
    assert len(finite) == 254


def test_e4m3_encode_roundtrips_every_finite_code():
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)


def _rounding_sweep():
    """fp32 patterns around every e4m3 rounding decision point in |f| < 512:
    for each fp32 exponent field and each value of the top 3 mantissa bits,
    the low 20 bits take values at, next to and around the halfway pattern."""
    lows = [0, 1, 2, 3, 0x7FFFD, 0x7FFFE, 0x7FFFF, 0x80000, 0x80001, 0x80002,
            0xFFFFD, 0xFFFFE, 0xFFFFF]
    rng = np.random.default_rng(1)
    lows += list(rng.integers(0, 1 << 20, 40))
    pats = []
    for exp_field in range(0, 0x88):
        for top in range(8):
            for low in lows:
                pats.append((exp_field << 23) | (top << 20) | int(low))
    pats = np.array(pats, dtype=np.uint32)
    pats = np.concatenate([pats, pats | np.uint32(0x80000000)])
    return pats.view(np.float32)


def test_e4m3_encode_matches_torch_cast_at_rounding_points():
    f = _rounding_sweep()
    f = f[np.abs(f) <= 464.0]     # torch maps anything that rounds past 448 to NaN
    assert np.array_equal(oracle.e4m3_encode_array(f), torch_e4m3_bytes(f))


def test_e4m3_encode_matches_torch_cast_random():
    rng = np.random.default_rng(2)
    mag = np.exp2(rng.uniform(-16, np.log2(464.0), 2_000_000)).astype(np.float32)
    sign = np.where(rng.random(mag.size) < 0.5, -1, 1).astype(np.float32)
    f = mag * sign
    f = f[np.abs(f) <= 464.0]
    assert np.array_equal(oracle.e4m3_encode_array(f), torch_e4m3_bytes(f))


def test_e4m3_encode_ties_to_even_and_saturates():
    # 464 is halfway between 448 (mantissa 110, even) and 480 (not representable)
    assert oracle.e4m3_encode(464.0) == 0x7E
    for v in (464.0001, 479.0, 480.0, 1e6, float("inf")):
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE
    assert oracle.e4m3_encode(float("nan")) & 0x7F == 0x7F
    # halfway between 1.0 (even) and 1.125 goes to 1.0; between 1.125 and 1.25 to 1.25
    assert oracle.e4m3_encode(1.0625) == 0x38
    assert oracle.e4m3_encode(1.1875) == 0x3A
    # below half the smallest subnormal -> zero, exactly half -> zero (even), above -> 2^-9
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00
    assert oracle.e4m3_encode(float(np.nextafter(f32(2.0 ** -10), f32(1)))) == 0x01
    assert oracle.e4m3_encode(-0.0) == 0x80


# --------------------------------------------------------------------------
# bf16 rounding
# --------------------------------------------------------------------------

def test_bf16_rne_matches_torch_cast():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 1 << 32, 400_000, dtype=np.uint64).astype(np.uint32)
    low = np.array([0x7FFF, 0x8000, 0x8001, 0x0000, 0xFFFF], dtype=np.uint32)
    edge = (bits[:5000, None] & np.uint32(0xFFFF0000)) | low[None, :]
    bits = np.concatenate([bits, edge.ravel()])
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ours = np.array([oracle.bf16_from_f32(v) for v in f[:100_000]], dtype=np.uint16)
    ref = torch.from_numpy(f[:100_000].copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------
# Scale rule
# --------------------------------------------------------------------------

def _exact_pow2_ceil(s):
    """2^ceil(log2 s) by exact rational comparison (independent of frexp)."""
    r = Fraction(float(s))
    e = 0
    while Fraction(2) ** e < r:
        e += 1
    while Fraction(2) ** (e - 1) >= r:
        e -= 1
    return float(Fraction(2) ** e)


def test_ue8m0_round_up_is_exact_power_of_two_ceiling():
    rng = np.random.default_rng(4)
    vals = np.exp2(rng.uniform(-30, 30, 3000)).astype(np.float32)
    vals = np.concatenate([vals, np.float32([1.0, 0.5, 2.0 ** -22, 1.5, 0.75,
                                             np.nextafter(f32(1), f32(2)),
                                             np.nextafter(f32(1), f32(0))])])
    for v in vals:
        assert oracle.ue8m0_round_up(v) == _exact_pow2_ceil(v), v
    # an infinite scale (a block holding inf) has no larger power of two
    assert oracle.ue8m0_round_up(np.inf) == np.inf
    assert oracle.block_scale(np.inf, True) == np.inf


def test_block_scale_pages_constants():
    # amax equal to the e4m3 maximum gives a unit scale
    assert oracle.block_scale(E4M3_MAX, False) == 1.0
    assert oracle.block_scale(E4M3_MAX, True) == 1.0
    # all-zero block: clamp to 1e-4 (fp32), then divide by 448 in fp32
    zero_s = f32(CLAMP) / f32(E4M3_MAX)
    assert oracle.block_scale(0.0, False) == zero_s
    assert oracle.block_scale(5e-5, False) == zero_s
    assert oracle.block_scale(0.0, True) == 2.0 ** -22   # 2.23e-7 lies in (2^-23, 2^-22]
    # above the clamp the scale is amax/448, one fp32 division
    assert oracle.block_scale(1.0, False) == f32(1.0) / f32(448.0)
    assert oracle.block_scale(449.0, True) == 2.0
    assert oracle.block_scale(224.0, True) == 0.5


# --------------------------------------------------------------------------
# act_quant
# --------------------------------------------------------------------------

def _bf16(x):
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_act_quant_pages_example_shapes():
    ex = FACTS["act_quant_example"]
    x = torch.randn(*ex["x_shape"], generator=torch.Generator().manual_seed(0))
    q, s = oracle.act_quant(x.numpy(), block=BLOCK)
    assert list(q.shape) == ex["q_shape"] and list(s.shape) == ex["s_shape"]


def test_act_quant_scales_are_per_1x128_block():
    x = torch.zeros(2, 4 * BLOCK)
    x[0, 5] = 1.0            # block 0 of row 0: amax 1
    x[0, BLOCK + 7] = -448.0  # block 1: amax 448 -> s = 1
    x[0, 2 * BLOCK] = 3.0    # block 2: amax 3
    # block 3 all zero -> clamp
    x[1, :] = 2.0
    q, s = oracle.act_quant(_bf16(x))
    zero_s = f32(CLAMP) / f32(E4M3_MAX)
    assert s[0, 0] == f32(1.0) / f32(448.0)
    assert s[0, 1] == 1.0
    assert s[0, 2] == f32(3.0) / f32(448.0)
    assert s[0, 3] == zero_s
    assert np.all(s[1] == f32(2.0) / f32(448.0))
    # the amax element of a block maps to +-448 (None format)
    assert q[0, 5] == 0x7E and q[0, BLOCK + 7] == 0xFE and q[0, 2 * BLOCK] == 0x7E
    assert np.all(q[1] == 0x7E)
    # zeros stay zeros
    assert np.all(q[0, 3 * BLOCK:] == 0)


def test_act_quant_unit_scale_block_is_plain_cast():
    # a block whose amax is exactly 448 has s = 1, so q is the plain cast of x
    rng = np.random.default_rng(5)
    x = rng.normal(0, 50, (8, BLOCK)).astype(np.float32)
    x = np.clip(x, -447, 447)
    x[:, 3] = 448.0
    xb = _bf16(torch.from_numpy(x))
    q, s = oracle.act_quant(xb)
    assert np.all(s == 1.0)
    xf = oracle.bf16_bits_to_f32(xb)
    assert np.array_equal(q, torch_e4m3_bytes(xf).reshape(q.shape))


def _dec(q):
    t = oracle.e4m3_table()
    return t[q]


def test_act_quant_invariants_and_roundtrip_bound():
    x = torch.randn(64, 8 * BLOCK, generator=torch.Generator().manual_seed(6))
    x[3, 100] = 300.0
    x[10, 129:140] = 1e-6
    x[20, 256:384] = 0.0
    for fmt in (None, "ue8m0"):
        xb = _bf16(x)
        q, s = oracle.act_quant(xb, scale_fmt=fmt)
        xf = oracle.bf16_bits_to_f32(xb).astype(np.float64).reshape(64, 8, BLOCK)
        d = _dec(q).reshape(64, 8, BLOCK)
        assert np.all(np.abs(d) <= E4M3_MAX)
        amax = np.abs(xf).max(axis=2)
        s_none = np.maximum(amax, f32(CLAMP)).astype(np.float32) / np.float32(448.0)
        if fmt is None:
            assert np.array_equal(s, s_none)
        else:
            m, _ = np.frexp(s)
            assert np.all(m == 0.5)                          # exact powers of two
            assert np.all(s >= s_none) and np.all(s < 2 * s_none)
        # |dec(q)*s - x| <= half an e4m3 step of x/s, times s (plus fp32 division rounding)
        y = xf / s[..., None]
        step = np.where(np.abs(y) < 2.0 ** -6, 2.0 ** -9,
                        np.exp2(np.floor(np.log2(np.maximum(np.abs(y), 1e-300))) - 3))
        err = np.abs(d * s[..., None] - xf)
        assert np.all(err <= (0.5 * step + np.abs(y) * 2.0 ** -23) * s[..., None] * (1 + 1e-12))


def test_act_quant_matches_library_division_and_cast():
    """q = cast_e4m3(fl32(x / s)) with torch's fp32 division and torch's cast."""
    x = torch.randn(32, 16 * BLOCK, generator=torch.Generator().manual_seed(7)) * 3
    x[torch.rand(x.shape, generator=torch.Generator().manual_seed(8)) < 0.01] *= 50
    for fmt in (None, "ue8m0"):
        for as_bf16 in (True, False):
            arr = _bf16(x) if as_bf16 else x.numpy()
            q, s = oracle.act_quant(arr, scale_fmt=fmt)
            xf = torch.from_numpy(oracle.bf16_bits_to_f32(arr) if as_bf16 else arr.copy())
            st = torch.from_numpy(s).repeat_interleave(BLOCK, dim=1)
            ref = (xf / st).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(q, ref)


@pytest.mark.parametrize("block", [32, 64, 256])
def test_act_quant_other_block_sizes_match_library_ops(block):
    """block_size is configurable: per 1 x block run, amax (torch max), the
    clamp and /448 in fp32, the ue8m0 round-up as an exact power-of-two
    ceiling (frexp), then torch's division and torch's e4m3 cast."""
    g = torch.Generator().manual_seed(block)
    x = torch.randn(24, 8 * block, generator=g) * 2
    x[torch.rand(x.shape, generator=g) < 0.02] *= 40
    x[3, :block] = 0.0                                   # an all-zero block
    for fmt in (None, "ue8m0"):
        q, s = oracle.act_quant(x.numpy(), block=block, scale_fmt=fmt)
        assert s.shape == (24, 8)
        amax = x.abs().reshape(24, 8, block).amax(dim=-1)
        a = torch.clamp(amax, min=float(f32(CLAMP)))
        sref = (a / torch.tensor(448.0)).numpy().astype(np.float32)
        if fmt == "ue8m0":
            m, e = np.frexp(sref.astype(np.float64))
            sref = np.where(m == 0.5, sref, np.ldexp(1.0, e)).astype(np.float32)
        assert np.array_equal(s.view(np.uint32), sref.view(np.uint32))
        st = torch.from_numpy(s).repeat_interleave(block, dim=1)
        ref = (x / st).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q, ref)


@pytest.mark.parametrize("block", [32, 64, 256])
def test_weight_dequant_other_block_sizes_match_library_ops(block):
    M, N = 2 * block + 5, 3 * block - 7
    g = torch.Generator().manual_seed(block + 1)
    codes = torch.randint(0, 254, (M, N), generator=g)
    codes = (codes + (codes >= 0x7F).long()).to(torch.uint8)
    rb, cb = -(-M // block), -(-N // block)
    s = torch.rand(rb, cb, generator=g) * (1e-3 - 1e-5) + 1e-5
    y = oracle.weight_dequant(codes.numpy(), s.numpy(), block=block)
    st = s.repeat_interleave(block, 0)[:M].repeat_interleave(block, 1)[:, :N]
    deq = codes.view(torch.float8_e4m3fn).float() * st
    assert np.array_equal(y, deq.bfloat16().view(torch.int16).numpy().view(np.uint16))


# --------------------------------------------------------------------------
# Test-data weight quantizer
# --------------------------------------------------------------------------

def test_weight_quant_tiles_and_ragged_edges():
    rng = np.random.default_rng(9)
    w = rng.normal(0, 0.02, (300, 576)).astype(np.float32)
    w[0, 0] = 448.0
    w[200:300, 512:576] = 0.0
    q, s = oracle.weight_quant(w)
    assert s.shape == (3, 5)                     # ceil(300/128), ceil(576/128)
    assert s[0, 0] == 1.0
    assert s[2, 4] == f32(CLAMP) / f32(E4M3_MAX)  # the all-zero ragged corner
    for bi in range(3):
        for bj in range(5):
            tile = w[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
            a = max(np.abs(tile).max(), f32(CLAMP))
            assert s[bi, bj] == np.float32(a) / np.float32(448.0)
            st = torch.from_numpy(tile.copy()) / float(s[bi, bj])
            ref = st.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(q[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128], ref)


@pytest.mark.parametrize("block", [32, 64, 128, 256])
def test_weight_quant_block_sizes_and_ue8m0_match_library_ops(block):
    """Per block x block tile (ragged at the bottom and right edges): amax by
    torch, the clamp and /448 in fp32, the ue8m0 round-up as an exact
    power-of-two ceiling, then torch's division and torch's e4m3 cast."""
    rows, cols = 2 * block + 9, 3 * block - 5
    g = torch.Generator().manual_seed(300 + block)
    w = torch.randn(rows, cols, generator=g) * 0.02
    w[torch.rand(w.shape, generator=g) < 0.01] *= 30
    w[block:2 * block, :block] = 0.0                      # an all-zero tile
    rb, cb = -(-rows // block), -(-cols // block)
    pad = torch.zeros(rb * block, cb * block)
    pad[:rows, :cols] = w.abs()
    amax = pad.reshape(rb, block, cb, block).amax(dim=(1, 3))
    s_none = (torch.clamp(amax, min=float(f32(CLAMP))) / torch.tensor(448.0)).numpy()
    for fmt in (None, "ue8m0"):
        q, s = oracle.weight_quant(w.numpy(), block=block, scale_fmt=fmt)
        sref = s_none.astype(np.float32)
        if fmt == "ue8m0":
            sref = np.array([_exact_pow2_ceil(v) for v in sref.ravel()],
                            dtype=np.float32).reshape(sref.shape)
        assert np.array_equal(s.view(np.uint32), sref.view(np.uint32)), fmt
        st = torch.from_numpy(s).repeat_interleave(block, 0)[:rows].repeat_interleave(block, 1)[:, :cols]
        ref = (w / st).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q, ref), fmt


# --------------------------------------------------------------------------
# weight_dequant
# --------------------------------------------------------------------------

def test_weight_dequant_pages_example_shape():
    ex = FACTS["weight_dequant_example"]
    q = np.zeros(ex["w_shape"], dtype=np.uint8)
    s = np.ones(ex["s_shape"], dtype=np.float32)
    y = oracle.weight_dequant(q, s)
    assert y.shape == tuple(ex["w_shape"])
    with pytest.raises(ValueError):
        oracle.weight_dequant(q, np.ones((7, 8), dtype=np.float32))


@pytest.mark.parametrize("shape", [(256, 256), (200, 576), (129, 130)])
def test_weight_dequant_matches_library_multiply_and_cast(shape):
    M, N = shape
    g = torch.Generator().manual_seed(10)
    codes = torch.randint(0, 254, (M, N), generator=g)
    codes = (codes + (codes >= 0x7F).long()).to(torch.uint8)
    rb, cb = -(-M // 128), -(-N // 128)
    s = torch.rand(rb, cb, generator=g) * (1e-3 - 1e-5) + 1e-5
    s[0, -1] = -3.5e-4      # any finite scale is accepted
    y = oracle.weight_dequant(codes.numpy(), s.numpy())
    y32 = oracle.weight_dequant(codes.numpy(), s.numpy(), out="f32")
    # element (i, j) takes the scale at (i // 128) * cdiv(N, 128) + j // 128
    st = s.repeat_interleave(128, 0)[:M].repeat_interleave(128, 1)[:, :N]
    prod = codes.view(torch.float8_e4m3fn).to(torch.float32) * st
    assert np.array_equal(y32, prod.numpy())
    ref = prod.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y, ref)


# --------------------------------------------------------------------------
# GEMM reference
# --------------------------------------------------------------------------

def _random_problem(M, N, K, seed, ue8m0=False):
    g = torch.Generator().manual_seed(seed)
    codes_a = torch.randint(0, 254, (M, K), generator=g)
    codes_a = (codes_a + (codes_a >= 0x7F).long()).to(torch.uint8).numpy()
    codes_w = torch.randint(0, 254, (N, K), generator=g)
    codes_w = (codes_w + (codes_w >= 0x7F).long()).to(torch.uint8).numpy()
    sa = (torch.rand(M, K // 128, generator=g) * 2 + 0.01).numpy().astype(np.float32)
    sw = (torch.rand(-(-N // 128), K // 128, generator=g) * 0.01 + 1e-4).numpy().astype(np.float32)
    if ue8m0:
        sa = np.exp2(np.round(np.log2(sa))).astype(np.float32)
        sw = np.exp2(np.round(np.log2(sw))).astype(np.float32)
    return codes_a, sa, codes_w, sw


def _exact_gemm(qa, sa, qw, sw, w_rows=128):
    """Exact y and bound with integer arithmetic: every e4m3 value times 2^9 is
    an integer, so each 128-wide partial sum is an integer times 2^-18; the
    scales are then applied as exact rationals.  Row n of W takes scale row
    n // w_rows (128: weight blocks; 1: per-row scales)."""
    table = oracle.e4m3_table()
    ia = np.rint(table[qa] * 512).astype(np.int64)
    iw = np.rint(table[qw] * 512).astype(np.int64)
    M, K = qa.shape
    N = qw.shape[0]
    y = [[Fraction(0)] * N for _ in range(M)]
    b = [[Fraction(0)] * N for _ in range(M)]
    for kb in range(K // 128):
        sl = slice(kb * 128, (kb + 1) * 128)
        P = ia[:, sl] @ iw[:, sl].T
        Pabs = np.abs(ia[:, sl]) @ np.abs(iw[:, sl]).T
        for m in range(M):
            fa = Fraction(float(sa[m, kb]))
            for n in range(N):
                sc = fa * Fraction(float(sw[n // w_rows, kb])) / (1 << 18)
                y[m][n] += sc * int(P[m, n])
                b[m][n] += abs(sc) * int(Pabs[m, n])
    return y, b


@pytest.mark.parametrize("M,N,K", [(3, 128, 128), (4, 256, 256), (2, 320, 384)])
def test_gemm_matches_exact_integer_arithmetic(M, N, K):
    qa, sa, qw, sw = _random_problem(M, N, K, seed=M * 1000 + N + K)
    y, bnd = oracle.gemm(qa, sa, qw, sw)
    ye, be = _exact_gemm(qa, sa, qw, sw)
    for m in range(M):
        for n in range(N):
            tol = float(be[m][n]) * 2.0 ** -50
            assert abs(Fraction(float(y[m, n])) - ye[m][n]) <= Fraction(tol), (m, n)
            assert abs(bnd[m, n] - float(be[m][n])) <= tol


def test_gemm_matches_library_matmul_tiny_config():
    # the tiny linear: x [128,512] ~N(0,1) with 1% outliers x50, W [256,512] ~N(0,0.02)
    from fp8_block_scaled_10_b200 import workloads as wl
    x = wl.normal_with_outliers(128, 512, seed=0, frac=0.01, factor=50.0)
    w = wl.weight_f32(256, 512, seed=1)
    qa, sa = oracle.act_quant(wl.bf16_bits(x))
    qw, sw = oracle.weight_quant(w.numpy())
    assert sw.shape == (2, 4)
    y, bnd = oracle.gemm(qa, sa, qw, sw)
    table = torch.from_numpy(oracle.e4m3_table())
    a_hat = table[torch.from_numpy(qa).long()] * torch.from_numpy(sa).double().repeat_interleave(128, 1)
    w_hat = table[torch.from_numpy(qw).long()] * \
        torch.from_numpy(sw).double().repeat_interleave(128, 0)[:256].repeat_interleave(128, 1)
    ref = (a_hat @ w_hat.T).numpy()
    ref_b = (a_hat.abs() @ w_hat.abs().T).numpy()
    assert np.all(np.abs(y - ref) <= 1e-12 * ref_b)
    assert np.allclose(bnd, ref_b, rtol=1e-12, atol=0)


def test_gemm_special_cases():
    # all-ones W with unit scales reduces y to the row sums of the dequantized A
    qa, sa, _, _ = _random_problem(5, 128, 256, seed=11)
    qw = np.full((128, 256), 0x38, dtype=np.uint8)     # e4m3 1.0
    sw = np.ones((1, 2), dtype=np.float32)
    y, _ = oracle.gemm(qa, sa, qw, sw)
    a_hat = oracle.e4m3_table()[qa] * np.repeat(sa.astype(np.float64), 128, axis=1)
    assert np.allclose(y, a_hat.sum(axis=1, keepdims=True).repeat(128, 1), rtol=1e-14, atol=1e-300)
    # a single nonzero K block isolates its (sa * sw) pair
    qa, sa, qw, sw = _random_problem(4, 256, 384, seed=12)
    qa[:, :128] = 0
    qa[:, 256:] = 0
    y, _ = oracle.gemm(qa, sa, qw, sw)
    t = oracle.e4m3_table()
    for m in range(4):
        for n in (0, 127, 128, 255):
            p = float(np.dot(t[qa[m, 128:256]], t[qw[n, 128:256]]))
            assert y[m, n] == float(sa[m, 1]) * float(sw[n // 128, 1]) * p
    # sign: negating A negates y exactly
    yn, _ = oracle.gemm(qa ^ np.uint8(0x80), sa, qw, sw)
    assert np.array_equal(yn, -y)


# --------------------------------------------------------------------------
# static activation scheme: precomputed scales, static_dequant
# --------------------------------------------------------------------------

def _static_case(rows, nblk, block, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, nblk * block, generator=g) * 2
    x[torch.rand(x.shape, generator=g) < 0.02] *= 300       # saturating entries
    s = torch.exp2(torch.rand(nblk, generator=g) * 8 - 6) * (1 + torch.rand(nblk, generator=g))
    return x, s.to(torch.float32)


def _torch_static_codes(x, st):
    """torch's fp32 division and e4m3 cast; where the rounded quotient lies at
    or beyond 464 (halfway from 448 to the next binade step, 480) torch gives
    NaN, and the saturating cast gives the signed maximum 448 (code 0x7E)."""
    y = x / st
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    big = (y.abs() >= 464).numpy()
    ref[big] = np.where(y.numpy()[big] < 0, 0xFE, 0x7E)
    return ref


@pytest.mark.parametrize("block", [128, 32, 256])
def test_act_quant_static_matches_library_division_and_cast(block):
    x, s = _static_case(20, 6, block, seed=block + 11)
    for as_bf16 in (False, True):
        arr = _bf16(x) if as_bf16 else x.numpy()
        xf = torch.from_numpy(oracle.bf16_bits_to_f32(arr) if as_bf16 else arr.copy())
        q = oracle.act_quant_static(arr, s.numpy(), block=block)
        st = s.repeat_interleave(block).unsqueeze(0).expand_as(xf)
        ref = _torch_static_codes(xf, st)
        assert np.array_equal(q, ref)
        assert ((q & 0x7F) == 0x7E).sum() > 0                # saturation was exercised


def test_act_quant_static_scale_index_is_the_channel_block():
    """x = 1 everywhere and s[b] = 2^-b: every row's block b holds 2^b, so a
    scale looked up by row, or by column modulo the block count, fails."""
    rows, nblk = 5, 7
    x = np.ones((rows, nblk * BLOCK), np.float32)
    s = np.exp2(-np.arange(nblk, dtype=np.float32)).astype(np.float32)
    q = oracle.act_quant_static(x, s)
    want = torch_e4m3_bytes(np.exp2(np.arange(nblk, dtype=np.float32)))
    assert np.array_equal(q, np.broadcast_to(np.repeat(want, BLOCK), q.shape))
    # and the per-row table form: row r uses s_tab[r, b]
    s_tab = np.stack([s * np.float32(2.0 ** r) for r in range(rows)]).astype(np.float32)
    q2 = oracle.act_quant_static(x, s_tab)
    for r in range(rows):
        want = torch_e4m3_bytes(np.exp2(np.arange(nblk, dtype=np.float32) - r))
        assert np.array_equal(q2[r], np.repeat(want, BLOCK))


def test_act_quant_static_with_dynamic_scales_is_act_quant():
    """Given the scales the dynamic scheme computes, as a per-row table, the
    static quantizer reproduces its codes (same division, same cast)."""
    x = torch.randn(33, 5 * BLOCK, generator=torch.Generator().manual_seed(21)) * 4
    arr = _bf16(x)
    for fmt in (None, "ue8m0"):
        q, s = oracle.act_quant(arr, scale_fmt=fmt)
        assert np.array_equal(oracle.act_quant_static(arr, s), q)


@pytest.mark.parametrize("block", [128, 64])
def test_act_dequant_matches_pages_static_dequant(block):
    """static_dequant as the page writes it: q_x.float() times the scales
    unsqueezed over the last axis (q viewed as [rows, blocks, block]), in
    torch fp32, then torch's bf16 cast; and with a per-row table."""
    rows, nblk = 9, 5
    g = torch.Generator().manual_seed(block + 5)
    codes = torch.randint(0, 254, (rows, nblk * block), generator=g)
    codes = (codes + (codes >= 0x7F).long()).to(torch.uint8)   # skip the NaN code 0x7F
    s = (torch.rand(nblk, generator=g) * 1e-2 + 1e-5).to(torch.float32)
    qf = codes.view(torch.float8_e4m3fn).float().reshape(rows, nblk, block)
    ref = (qf * s.unsqueeze(-1)).reshape(rows, -1)
    y32 = oracle.act_dequant(codes.numpy(), s.numpy(), block=block, out="f32")
    assert np.array_equal(y32.view(np.uint32), ref.numpy().view(np.uint32))
    y16 = oracle.act_dequant(codes.numpy(), s.numpy(), block=block)
    assert np.array_equal(y16, ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    s_tab = (torch.rand(rows, nblk, generator=g) * 3 + 0.1).to(torch.float32)
    ref = (qf * s_tab.unsqueeze(-1)).reshape(rows, -1)
    y32 = oracle.act_dequant(codes.numpy(), s_tab.numpy(), block=block, out="f32")
    assert np.array_equal(y32.view(np.uint32), ref.numpy().view(np.uint32))


# --------------------------------------------------------------------------
# training GEMMs: per-row scales on both operands, transposed operands
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(3, 130, 128), (2, 257, 384)])
def test_gemm_row_scaled_b_matches_exact_integer_arithmetic(M, N, K):
    """One scale per row of the second operand and K block (w_scales="row")."""
    qa, sa, qw, _ = _random_problem(M, N, K, seed=M * 7 + N + K)
    g = torch.Generator().manual_seed(N)
    sb = (torch.rand(N, K // 128, generator=g) * 0.5 + 1e-3).numpy().astype(np.float32)
    y, bnd = oracle.gemm(qa, sa, qw, sb, w_scales="row")
    ye, be = _exact_gemm(qa, sa, qw, sb, w_rows=1)
    for m in range(M):
        for n in range(N):
            tol = float(be[m][n]) * 2.0 ** -50
            assert abs(Fraction(float(y[m, n])) - ye[m][n]) <= Fraction(tol), (m, n)
            assert abs(bnd[m, n] - float(be[m][n])) <= tol


def test_gemm_row_scales_equal_to_block_scales_agree():
    """Row scales that repeat each weight block's scale over its 128 rows
    give the block-scaled result exactly."""
    qa, sa, qw, sw = _random_problem(5, 300, 256, seed=31)
    y_blk, _ = oracle.gemm(qa, sa, qw, sw)
    y_row, _ = oracle.gemm(qa, sa, qw, np.repeat(sw, 128, axis=0)[:300].copy(), w_scales="row")
    assert np.array_equal(y_blk, y_row)


def test_act_quant_transposed_matches_library_ops():
    """128 x 1 column blocks of x (amax over 128 consecutive rows of one
    column, by torch on x itself, no transpose), torch's division and cast,
    then the result laid out transposed."""
    g = torch.Generator().manual_seed(41)
    R, C = 3 * BLOCK, 200
    x = torch.randn(R, C, generator=g) * 3
    x[torch.rand(x.shape, generator=g) < 0.01] *= 60
    x[:BLOCK, 7] = 0.0                                  # an all-zero column block
    arr = _bf16(x)
    xf = torch.from_numpy(oracle.bf16_bits_to_f32(arr).copy())
    for fmt in (None, "ue8m0"):
        q, s = oracle.act_quant_transposed(arr, scale_fmt=fmt)
        assert q.shape == (C, R) and s.shape == (C, R // BLOCK)
        amax = xf.abs().reshape(R // BLOCK, BLOCK, C).amax(dim=1)          # [R/128, C]
        a = torch.clamp(amax, min=float(f32(CLAMP)))
        sref = (a / torch.tensor(448.0)).numpy().astype(np.float32)
        if fmt == "ue8m0":
            m, e = np.frexp(sref.astype(np.float64))
            sref = np.where(m == 0.5, sref, np.ldexp(1.0, e)).astype(np.float32)
        assert np.array_equal(s.view(np.uint32), sref.T.view(np.uint32))
        st = torch.from_numpy(sref).repeat_interleave(BLOCK, dim=0)        # [R, C]
        ref = (xf / st).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q, ref.T)


def test_weight_gradient_gemm_matches_library_matmul():
    """dW = dy^T x with both operands quantized in 128 x 1 blocks along the
    token dimension: the row-scaled GEMM of the transposed operands equals
    torch's float64 matmul of the dequantized dy and x."""
    g = torch.Generator().manual_seed(43)
    T, N, K = 256, 192, 136                       # tokens, out features, in features
    dy = torch.randn(T, N, generator=g) * 1e-2
    x = torch.randn(T, K, generator=g)
    qd, sd = oracle.act_quant_transposed(_bf16(dy))            # [N, T], [N, T/128]
    qx, sx = oracle.act_quant_transposed(_bf16(x))             # [K, T], [K, T/128]
    dw, bnd = oracle.gemm(qd, sd, qx, sx, w_scales="row")       # [N, K]
    t = torch.from_numpy(oracle.e4m3_table())
    d_hat = t[torch.from_numpy(qd).long()] * torch.from_numpy(sd).double().repeat_interleave(BLOCK, 1)
    x_hat = t[torch.from_numpy(qx).long()] * torch.from_numpy(sx).double().repeat_interleave(BLOCK, 1)
    ref = (d_hat @ x_hat.T).numpy()                             # dy_hat^T x_hat, [N, K]
    assert np.all(np.abs(dw - ref) <= 1e-12 * bnd)


def test_fp8_transpose_and_dequant_commute():
    """dequant(q^T, s^T) is the transpose of dequant(q, s), on ragged shapes,
    and transposing twice is the identity."""
    g = torch.Generator().manual_seed(47)
    R, C = 300, 200
    codes = torch.randint(0, 254, (R, C), generator=g)
    codes = (codes + (codes >= 0x7F).long()).to(torch.uint8).numpy()
    s = (torch.rand(3, 2, generator=g) + 0.01).numpy().astype(np.float32)
    qt, st = oracle.fp8_transpose(codes, s)
    assert qt.shape == (C, R) and st.shape == (2, 3)
    y = oracle.weight_dequant(codes, s, out="f32")
    yt = oracle.weight_dequant(qt, st, out="f32")
    assert np.array_equal(yt, y.T)
    q2, s2 = oracle.fp8_transpose(qt, st)
    assert np.array_equal(q2, codes) and np.array_equal(s2, s)
