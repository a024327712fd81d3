"""The seeded input generators follow the input recipe (CPU): the same seed
gives the same bits, and each generator's draws have the stated structure
(outlier fraction and scale, the number of Student-t channels, the weight
spread, the finite e4m3 codes, multinomial expert counts)."""
import numpy as np
import torch

from fp8_block_scaled_10_b200 import workloads as wl


def test_same_seed_same_bits():
    for f in (lambda s: wl.normal_with_outliers(64, 256, s, 0.01, 50.0),
              lambda s: wl.heavy_tailed_channels(64, 256, s),
              lambda s: wl.weight_f32(64, 256, s),
              lambda s: wl.e4m3_codes(64, 256, s),
              lambda s: wl.uniform((64,), 0.01, 0.5, s),
              lambda s: wl.expert_counts(4096, 32, s)):
        a, b, c = f(7), f(7), f(8)
        assert torch.equal(a, b)
        assert not torch.equal(a, c)


def test_normal_with_outliers_fraction_and_scale():
    x = wl.normal_with_outliers(4096, 512, seed=1, frac=0.01, factor=50.0).float()
    big = (x.abs() > 10).float().mean().item()
    # outliers are N(0, 50^2): |x| > 10 for 84 % of them, and for no N(0,1) entry
    assert 0.0070 < big < 0.0100, big
    assert x.abs().max().item() > 100


def test_heavy_tailed_channels_count_and_tails():
    x = wl.heavy_tailed_channels(4096, 7168, seed=2).float()
    col_max = x.abs().amax(dim=0)
    heavy = int((col_max > 7).sum().item())
    assert heavy == round(0.01 * 7168), heavy          # 72 Student-t(3) channels
    normal = col_max[col_max <= 7]
    assert normal.max().item() < 6.5                     # the N(0,1) channels have light tails


def test_weight_spread_and_codes():
    w = wl.weight_f32(2048, 2048, seed=3)
    assert abs(w.std().item() - 0.02) < 0.0005 and abs(w.mean().item()) < 0.0005
    q = wl.e4m3_codes(1024, 1024, seed=4).numpy()
    counts = np.bincount(q.ravel(), minlength=256)
    assert counts[0x7F] == 0 and counts[0xFF] == 0
    finite = np.delete(counts, [0x7F, 0xFF])
    assert finite.min() > 0.8 * finite.mean() and finite.max() < 1.2 * finite.mean()


def test_expert_counts_are_multinomial():
    c = wl.expert_counts(wl.EXPERT_TOKENS * wl.EXPERT_TOPK, wl.EXPERTS, seed=70)
    assert c.dtype == torch.int64 and c.numel() == wl.EXPERTS
    assert int(c.sum()) == wl.EXPERT_TOKENS * wl.EXPERT_TOPK == 65536
    mean = 65536 / 32
    assert (c.float() - mean).abs().max().item() < 5 * mean ** 0.5   # ~5 sigma


def test_uniform_range():
    u = wl.uniform((100000,), 0.01, 0.5, seed=5)
    assert u.min().item() >= 0.01 and u.max().item() < 0.5
    assert abs(u.mean().item() - 0.255) < 0.005
