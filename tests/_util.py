"""Helpers shared by the GPU parity tests: input preparation on the CPU (seeded
generators + the oracle) and the GEMM tolerance check."""
import numpy as np
import torch

import oracle
from fp8_block_scaled_10_b200 import workloads as wl

GEMM_REL = 4e-3
GEMM_ABS_OF_BOUND = 1e-3


def u8(t):
    return t.view(torch.uint8).cpu().numpy()


def f32bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def cuda_codes(q_np):
    return torch.from_numpy(np.ascontiguousarray(q_np)).cuda().view(torch.float8_e4m3fn)


def cuda_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def quantized_weight(N, K, seed, scale_fmt=None):
    """W ~N(0, 0.02) [N, K] fp32, quantized per 128x128 block by the oracle."""
    w = wl.weight_f32(N, K, seed=seed).numpy()
    return oracle.weight_quant(w, scale_fmt=scale_fmt)


def assert_gemm_close(y_gpu, y_ref, bound, what=""):
    """|y - y_ref| <= 4e-3 |y_ref| + 1e-3 sum_k |a_k w_k| element-wise."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    err = np.abs(y - y_ref)
    tol = GEMM_REL * np.abs(y_ref) + GEMM_ABS_OF_BOUND * bound
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        detail = ", ".join("(%d,%d): gpu %.6g ref %.6g tol %.3g" % (i, j, y[i, j], y_ref[i, j], tol[i, j])
                           for i, j in idx)
        raise AssertionError("%s: %d of %d outside tolerance; first %s"
                             % (what, int(bad.sum()), bad.size, detail))
    return float((err / np.maximum(tol, 1e-300)).max())


def sample_rows(M, n_random, seed):
    """Rows at every 128-row tile edge near the start and end, plus random rows."""
    rows = {0, 1, 126, 127, 128, 129, M - 1, M - 2, M - 128, M - 129, M // 2}
    rng = np.random.default_rng(seed)
    rows |= set(int(r) for r in rng.integers(0, M, n_random))
    return np.array(sorted(r for r in rows if 0 <= r < M), dtype=np.int64)
