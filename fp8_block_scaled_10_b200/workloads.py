"""Seeded synthetic inputs for the FP8 block-scaled linear workloads.

This module only draws random numbers and names shapes; it holds none of the
quantization or GEMM arithmetic.  The CUDA path (tests, benchmark) and the CPU
oracle (tests, CPU baseline) both take their inputs from here, so that the two
sides see identical data when the generator runs on the CPU.  Generators
accept ``device``; numbers drawn on a CUDA device differ from the CPU stream
for the same seed (the benchmark draws on the device to save time and never
compares against the oracle bit for bit).

Workloads (DeepSeek-V3 layer shapes: hidden 7168, dense FFN 18432, expert FFN
2048, the 576-wide ragged projection):

* ``tiny``      x bf16 [128,512] ~N(0,1) with 1% of entries x50; W [256,512]
                ~N(0,0.02) quantized per 128x128 block; y bf16 [128,256].
* ``memory``    act_quant of x bf16 [16384,7168] ~N(0,1) with 0.1% entries
                x100; weight_dequant of e4m3 W [18432,7168] (uniform over the
                254 finite codes), scales [144,56] ~U(1e-5,1e-3).
* ``decode``    M in {1,8,32,64}; (K,N) = (7168,18432) and (18432,7168).
* ``prefill``   M=4096; (K,N) = (7168,18432), (18432,7168), (7168,576);
                x ~N(0,1) with 1% of channels Student-t (nu=3).
* ``experts``   32 experts, W_e [2048,7168]; 65536 routed rows, counts
                ~Multinomial(65536, uniform 1/32).
"""
import torch

HIDDEN = 7168
FFN = 18432
EXPERT_FFN = 2048
RAGGED_N = 576

DECODE_M = (1, 8, 32, 64)
DECODE_KN = ((7168, 18432), (18432, 7168))
PREFILL_M = 4096
PREFILL_KN = ((7168, 18432), (18432, 7168), (7168, 576))
EXPERTS = 32
EXPERT_TOKENS = 8192
EXPERT_TOPK = 8


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_with_outliers(rows, cols, seed, frac, factor, device="cpu", dtype=torch.bfloat16):
    """N(0,1) entries; a seeded Bernoulli(frac) subset is multiplied by factor."""
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    if frac > 0:
        mask = torch.rand(rows, cols, generator=g, device=device) < frac
        x = torch.where(mask, x * factor, x)
    return x.to(dtype)


def heavy_tailed_channels(rows, cols, seed, channel_frac=0.01, nu=3, device="cpu",
                          dtype=torch.bfloat16):
    """N(0,1) entries except a seeded subset of round(channel_frac*cols) columns,
    whose entries are Student-t with nu degrees of freedom, drawn as
    z0 / sqrt(chi2_nu / nu) with chi2_nu a sum of nu squared normals."""
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    nch = max(1, int(round(channel_frac * cols)))
    ch = torch.randperm(cols, generator=g, device=device)[:nch]
    z0 = torch.randn(rows, nch, generator=g, device=device)
    chi2 = torch.zeros(rows, nch, device=device)
    for _ in range(int(nu)):
        chi2 += torch.randn(rows, nch, generator=g, device=device) ** 2
    x[:, ch] = z0 / torch.sqrt(chi2 / nu)
    return x.to(dtype)


def weight_f32(rows, cols, seed, std=0.02, device="cpu"):
    """Dense fp32 weight ~N(0, std^2) (quantized per 128x128 block by the caller)."""
    g = _gen(seed, device)
    return torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std


def e4m3_codes(rows, cols, seed, device="cpu"):
    """uint8 codes drawn uniformly over the 254 finite e4m3fn codes (the two NaN
    codes 0x7F and 0xFF are skipped)."""
    g = _gen(seed, device)
    r = torch.randint(0, 254, (rows, cols), generator=g, device=device, dtype=torch.int32)
    r = r + (r >= 0x7F).to(torch.int32)          # skip 0x7F
    r = r + (r >= 0xFF).to(torch.int32)          # cannot happen: 253+1 = 254 < 255
    return r.to(torch.uint8)


def uniform(shape, lo, hi, seed, device="cpu"):
    g = _gen(seed, device)
    return torch.rand(*shape, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


def expert_counts(total, experts, seed):
    """Per-expert row counts ~Multinomial(total, uniform over experts), on the CPU."""
    g = _gen(seed, "cpu")
    idx = torch.randint(0, experts, (total,), generator=g)
    return torch.bincount(idx, minlength=experts).to(torch.int64)


def bf16_bits(t):
    """View a bf16 tensor's storage as int16 -> numpy uint16 bit patterns (CPU)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")
