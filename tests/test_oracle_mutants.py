"""Planted mistakes: each test takes an oracle result, plants a plausible slip
in it (on the CPU, in numpy), and checks that the reference comparison the
corresponding pin in test_oracle_pins.py relies on rejects the slipped
result while accepting the oracle's own.  This shows that the pins of
act_quant, weight_dequant and the GEMM, and those of the static scheme, the
transposing quantizer, the FP8 transpose and the row-scaled GEMM,
discriminate the slips they are meant to catch."""
from fractions import Fraction

import numpy as np
import torch

import oracle

BLOCK = 128


def _bf16(x):
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _torch_codes(y):
    return y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_static_scale_indexed_by_row_is_caught():
    """The static scale of element (r, c) is s[c // block]; a slip that reads
    s[r % nblk] instead is rejected by the x = 1, s[b] = 2^-b check."""
    rows, nblk = 5, 7
    x = np.ones((rows, nblk * BLOCK), np.float32)
    s = np.exp2(-np.arange(nblk, dtype=np.float32)).astype(np.float32)
    want = np.broadcast_to(np.repeat(_torch_codes(torch.from_numpy(1.0 / s)), BLOCK),
                           (rows, nblk * BLOCK))
    good = oracle.act_quant_static(x, s)
    assert np.array_equal(good, want)
    slip = np.stack([oracle.act_quant_static(x[r:r + 1], np.full(nblk, s[r % nblk], np.float32))[0]
                     for r in range(rows)])
    assert not np.array_equal(slip, want)


def test_static_dequant_without_scale_is_caught():
    """static_dequant multiplies by the block's scale; dropping it (or
    dividing) fails the page-formula comparison."""
    g = torch.Generator().manual_seed(3)
    codes = torch.randint(0, 254, (4, 2 * BLOCK), generator=g)
    codes = (codes + (codes >= 0x7F).long()).to(torch.uint8)
    s = torch.tensor([0.25, 3.0], dtype=torch.float32)
    ref = (codes.view(torch.float8_e4m3fn).float().reshape(4, 2, BLOCK) * s.unsqueeze(-1)).reshape(4, -1)
    good = oracle.act_dequant(codes.numpy(), s.numpy(), out="f32")
    assert np.array_equal(good, ref.numpy())
    for slip in (good / np.repeat(s.numpy(), BLOCK) ** 2, codes.view(torch.float8_e4m3fn).float().numpy()):
        assert not np.array_equal(slip.astype(np.float32), ref.numpy())


def test_transposed_quantizer_with_row_blocks_is_caught():
    """act_quant_transposed takes 128 x 1 column blocks; transposing the codes
    of ordinary 1 x 128 row blocks instead fails the column-block comparison."""
    g = torch.Generator().manual_seed(5)
    R, C = 2 * BLOCK, 2 * BLOCK
    x = torch.randn(R, C, generator=g) * 3
    x[torch.rand(x.shape, generator=g) < 0.02] *= 40
    arr = _bf16(x)
    xf = torch.from_numpy(oracle.bf16_bits_to_f32(arr).copy())
    amax = xf.abs().reshape(R // BLOCK, BLOCK, C).amax(dim=1)
    s = (torch.clamp(amax, min=float(np.float32(1e-4))) / torch.tensor(448.0)).numpy()
    want = _torch_codes(xf / torch.from_numpy(s).repeat_interleave(BLOCK, dim=0)).T
    good, _ = oracle.act_quant_transposed(arr)
    assert np.array_equal(good, want)
    slip = oracle.act_quant(arr)[0].T
    assert not np.array_equal(slip, want)


def test_fp8_transpose_without_scale_transpose_is_caught():
    """Transposing the codes with a scale grid of the right shape but its
    blocks in the wrong places fails the dequant-commutes check."""
    g = torch.Generator().manual_seed(7)
    codes = torch.randint(0, 254, (300, 200), generator=g)
    codes = (codes + (codes >= 0x7F).long()).to(torch.uint8).numpy()
    s = (torch.rand(3, 2, generator=g) + 0.01).numpy().astype(np.float32)
    y = oracle.weight_dequant(codes, s, out="f32")
    qt, st = oracle.fp8_transpose(codes, s)
    assert np.array_equal(oracle.weight_dequant(qt, st, out="f32"), y.T)
    flipped = np.ascontiguousarray(s[::-1, ::-1].T)   # right shape, wrong blocks
    assert not np.array_equal(oracle.weight_dequant(qt, flipped, out="f32"), y.T)


def test_row_scaled_gemm_with_block_scales_is_caught():
    """The row-scaled GEMM takes b_s[n, kb]; reading the scale of n's
    128-row block instead (b_s[n // 128 * 128, kb]) breaks exact arithmetic."""
    g = torch.Generator().manual_seed(9)
    M, N, K = 2, 130, 256
    qa = (torch.randint(0, 126, (M, K), generator=g)).to(torch.uint8).numpy()
    qb = (torch.randint(0, 126, (N, K), generator=g)).to(torch.uint8).numpy()
    sa = (torch.rand(M, K // 128, generator=g) + 0.5).numpy().astype(np.float32)
    sb = (torch.rand(N, K // 128, generator=g) + 0.5).numpy().astype(np.float32)
    y, _ = oracle.gemm(qa, sa, qb, sb, w_scales="row")
    table = oracle.e4m3_table()

    def exact(scales_for_row):
        out = np.zeros((M, N), dtype=object)
        for m in range(M):
            for n in range(N):
                acc = Fraction(0)
                for kb in range(K // 128):
                    sl = slice(kb * 128, (kb + 1) * 128)
                    p = sum(Fraction(float(a)) * Fraction(float(b))
                            for a, b in zip(table[qa[m, sl]], table[qb[n, sl]]))
                    acc += Fraction(float(sa[m, kb])) * Fraction(float(scales_for_row(n)[kb])) * p
                out[m, n] = acc
        return out

    ex = exact(lambda n: sb[n])
    assert all(abs(Fraction(float(y[m, n])) - ex[m, n]) <= abs(ex[m, n]) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)
               for m in range(M) for n in range(N))
    slip = exact(lambda n: sb[(n // 128) * 128])
    assert any(abs(Fraction(float(y[m, n])) - slip[m, n]) > abs(slip[m, n]) * Fraction(1, 2 ** 20)
               for m in range(M) for n in range(N))


# --------------------------------------------------------------------------
# the three functions of the forward path
# --------------------------------------------------------------------------

from test_oracle_pins import _exact_gemm, _random_problem  # noqa: E402


def _gemm_slip(qa, sa, qw, sw, scale):
    """y = sum_kb scale(m, n, kb) * (A_kb . W_kb^T) in float64: a GEMM with the
    given (possibly wrong) per-block scale product."""
    t = oracle.e4m3_table()
    a, w = t[qa], t[qw]
    M, K = qa.shape
    N = qw.shape[0]
    y = np.zeros((M, N))
    for kb in range(K // 128):
        sl = slice(kb * 128, (kb + 1) * 128)
        P = a[:, sl] @ w[:, sl].T
        for m in range(M):
            for n in range(N):
                y[m, n] += scale(m, n, kb) * P[m, n]
    return y


def _fails_exact_pin(y, ye, be):
    M, N = y.shape
    return any(abs(Fraction(float(y[m, n])) - ye[m][n]) > Fraction(float(be[m][n]) * 2.0 ** -50)
               for m in range(M) for n in range(N))


def test_gemm_slips_fail_the_exact_arithmetic_pin():
    """On the pin's non-trivial 2 x 320 x 384 problem (a 3 x 3 weight-scale
    grid), the exact comparison accepts the oracle and rejects: a transposed
    weight-scale index, a dropped activation scale, a weight-scale row taken
    as n modulo the grid's rows instead of n // 128, and one scale product
    for all K blocks (no per-block promotion)."""
    qa, sa, qw, sw = _random_problem(2, 320, 384, seed=2 * 1000 + 320 + 384)
    ye, be = _exact_gemm(qa, sa, qw, sw)
    y, _ = oracle.gemm(qa, sa, qw, sw)
    assert not _fails_exact_pin(y, ye, be)
    slips = {
        "transposed sw index": lambda m, n, kb: float(sa[m, kb]) * float(sw[kb, n // 128]),
        "dropped sa": lambda m, n, kb: float(sw[n // 128, kb]),
        "sw row n % rows": lambda m, n, kb: float(sa[m, kb]) * float(sw[n % sw.shape[0], kb]),
        "no per-block promotion": lambda m, n, kb: float(sa[m, 0]) * float(sw[n // 128, 0]),
    }
    for name, scale in slips.items():
        assert _fails_exact_pin(_gemm_slip(qa, sa, qw, sw, scale), ye, be), name


def test_act_quant_reciprocal_multiply_fails_the_division_pin():
    """q takes fl32(x / s); multiplying by fl32(1 / s) instead rounds
    differently on some elements of the pin's input, and the cast shows it."""
    x = torch.randn(32, 16 * BLOCK, generator=torch.Generator().manual_seed(7)) * 3
    x[torch.rand(x.shape, generator=torch.Generator().manual_seed(8)) < 0.01] *= 50
    arr = _bf16(x)
    q, s = oracle.act_quant(arr)
    xf = torch.from_numpy(oracle.bf16_bits_to_f32(arr).copy())
    st = torch.from_numpy(s).repeat_interleave(BLOCK, dim=1)
    ref = _torch_codes(xf / st)
    assert np.array_equal(q, ref)
    assert not np.array_equal(_torch_codes(xf * (1.0 / st)), ref)


def test_act_quant_scale_slips_fail_their_pins():
    """A ue8m0 scale rounded down, and a scale without the 1e-4 floor, break
    the invariant s_none <= s < 2 s_none and the all-zero block's value."""
    x = torch.randn(64, 8 * BLOCK, generator=torch.Generator().manual_seed(6))
    x[20, 256:384] = 0.0
    xb = _bf16(x)
    xf = oracle.bf16_bits_to_f32(xb).astype(np.float64).reshape(64, 8, BLOCK)
    amax = np.abs(xf).max(axis=2)
    s_none = np.maximum(amax, np.float32(1e-4)).astype(np.float32) / np.float32(448.0)
    _, s = oracle.act_quant(xb, scale_fmt="ue8m0")
    assert np.all(s >= s_none) and np.all(s < 2 * s_none)
    m, e = np.frexp(s_none)
    floor = np.ldexp(np.float32(0.5), e).astype(np.float32)
    floor[m == 0.5] = s_none[m == 0.5]
    assert not np.all(floor >= s_none)
    _, s_plain = oracle.act_quant(xb)
    unclamped = amax.astype(np.float32) / np.float32(448.0)
    assert s_plain[20, 2] == np.float32(1e-4) / np.float32(448.0)
    assert unclamped[20, 2] != s_plain[20, 2]


def test_weight_dequant_transposed_scale_index_fails_the_library_pin():
    """On a 256 x 576 weight (a 2 x 5 scale grid), scales indexed by the
    128-column block first and the row block second fail the torch multiply."""
    g = torch.Generator().manual_seed(10)
    codes = torch.randint(0, 254, (256, 576), generator=g)
    codes = (codes + (codes >= 0x7F).long()).to(torch.uint8)
    s = torch.rand(2, 5, generator=g) * (1e-3 - 1e-5) + 1e-5
    y32 = oracle.weight_dequant(codes.numpy(), s.numpy(), out="f32")
    st = s.repeat_interleave(128, 0).repeat_interleave(128, 1)[:, :576]
    ref = (codes.view(torch.float8_e4m3fn).to(torch.float32) * st).numpy()
    assert np.array_equal(y32, ref)
    flat = s.reshape(-1)
    i = torch.arange(256).unsqueeze(1) // 128
    j = torch.arange(576).unsqueeze(0) // 128
    wrong = flat[(j * 2 + i) % flat.numel()]        # column-major walk of the grid
    slip = (codes.view(torch.float8_e4m3fn).to(torch.float32) * wrong).numpy()
    assert not np.array_equal(slip, ref)


def test_weight_quant_with_row_blocks_is_caught():
    """weight_quant scales each 128 x 128 tile; quantizing in act_quant's
    1 x 128 row blocks instead fails the per-tile torch comparison."""
    g = torch.Generator().manual_seed(11)
    rows, cols = 2 * BLOCK + 9, 3 * BLOCK - 5
    w = torch.randn(rows, cols, generator=g) * 0.02
    w[torch.rand(w.shape, generator=g) < 0.01] *= 30
    rb, cb = -(-rows // BLOCK), -(-cols // BLOCK)
    pad = torch.zeros(rb * BLOCK, cb * BLOCK)
    pad[:rows, :cols] = w.abs()
    amax = pad.reshape(rb, BLOCK, cb, BLOCK).amax(dim=(1, 3))
    s = torch.clamp(amax, min=float(np.float32(1e-4))) / torch.tensor(448.0)
    st = s.repeat_interleave(BLOCK, 0)[:rows].repeat_interleave(BLOCK, 1)[:, :cols]
    want = _torch_codes(w / st)
    good, _ = oracle.weight_quant(w.numpy())
    assert np.array_equal(good, want)
    slip = np.concatenate([oracle.act_quant(np.ascontiguousarray(w[:, j:j + BLOCK].numpy()))[0]
                           for j in range(0, cols - cols % BLOCK, BLOCK)], axis=1)
    assert not np.array_equal(slip, want[:, :slip.shape[1]])
