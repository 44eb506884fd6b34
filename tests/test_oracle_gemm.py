"""Pins for the oracle's reference GEMM (fp64 product of the dequantized operands).

  * closed form: constant codes and per-tensor scales give C = K * value^2 * sA * sB;
  * numpy's float64 matmul (a library routine) on operands dequantized here with torch's
    float8 decode and explicitly expanded scale maps (repeat / kron), on non-square shapes
    so a transposed operand or a swapped scale index fails;
  * the page's identity y = sum_j s_x,j s_w,j (x_hat^(j) W_hat^(j)): the same product
    evaluated block by block over 128-wide K slices from raw codes, scales applied per block.
"""
import numpy as np
import pytest
import torch

import synth

TORCH_T = {0: torch.float8_e4m3fn, 1: torch.float8_e5m2}


def dec(codes, fmt=0):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(TORCH_T[fmt]).double().numpy()


def expand_a(sa, ga, M, K):
    return np.full((M, K), sa[0], np.float64) if ga == 0 else np.repeat(sa.T.astype(np.float64), 128, axis=1)[:, :K]


def expand_b(sb, gb, N, K):
    if gb == 0:
        return np.full((N, K), sb[0], np.float64)
    return np.kron(sb.astype(np.float64), np.ones((128, 128)))[:N, :K]


def make_operands(orc, M, N, K, ga, gb, seed):
    x = synth.activations(seed=seed, m=M, k=K)
    w = synth.weight_8b(seed=seed, n=N, k=K)
    a, sa = orc.quantize(x, orc.E4M3, orc.PER_TENSOR if ga == 0 else orc.GROUP_1x128)
    b, sb = orc.quantize(w, orc.E4M3, orc.PER_TENSOR if gb == 0 else orc.BLOCK_128x128)
    return a, sa, b, sb


def test_closed_form_constant_operands(orc):
    M, N, K = 3, 5, 384
    a = np.full((M, K), 0x38, np.uint8)          # 1.0
    b = np.full((N, K), 0x40, np.uint8)          # 2.0
    sa, sb = np.array([0.25], np.float32), np.array([3.0], np.float32)
    c = orc.gemm_rows(a, sa, 0, b, sb, 0, np.arange(M))
    assert np.all(c == K * 1.0 * 2.0 * 0.25 * 3.0)
    # a single nonzero block in K under block scales picks exactly that block's scales
    a2 = np.zeros((M, K), np.uint8); a2[:, 128:256] = 0x38
    sa2 = np.arange(1, 3 * M + 1, dtype=np.float32).reshape(3, M)
    sb2 = np.arange(1, 4, dtype=np.float32).reshape(1, 3) * 10
    c2 = orc.gemm_rows(a2, sa2, 1, b, sb2, 2, np.arange(M))
    for m in range(M):
        assert np.all(c2[m] == 128 * 2.0 * sa2[1, m] * sb2[0, 1])


@pytest.mark.parametrize("ga,gb", [(1, 2), (0, 0), (1, 0), (0, 2)])
@pytest.mark.parametrize("shape", [(7, 256, 384), (130, 384, 256), (1, 128, 128)])
def test_matches_numpy_matmul(orc, ga, gb, shape):
    M, N, K = shape
    a, sa, b, sb = make_operands(orc, M, N, K, ga, gb, seed=11)
    A = dec(a) * expand_a(sa, ga, M, K)
    B = dec(b) * expand_b(sb, gb, N, K)
    ref = A @ B.T
    rows = np.arange(M)
    got = orc.gemm_rows(a, sa, ga, b, sb, gb, rows)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_blockwise_identity(orc):
    """sum over K-blocks j of sA[j][m] * sB[n/128][j] * (codes_a^(j) . codes_b^(j))."""
    M, N, K = 9, 256, 512
    a, sa, b, sb = make_operands(orc, M, N, K, 1, 2, seed=12)
    Ac, Bc = dec(a), dec(b)
    y = np.zeros((M, N))
    for j in range(K // 128):
        ks = slice(j * 128, j * 128 + 128)
        part = Ac[:, ks] @ Bc[:, ks].T                                   # FP8 block product
        y += sa[j][:, None].astype(np.float64) * np.repeat(sb[:, j].astype(np.float64), 128)[None, :N] * part
    got = orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M))
    assert np.allclose(got, y, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_row_subset(orc):
    M, N, K = 40, 128, 256
    a, sa, b, sb = make_operands(orc, M, N, K, 1, 2, seed=13)
    full = orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M))
    rows = np.array([39, 0, 17, 17])
    assert np.array_equal(orc.gemm_rows(a, sa, 1, b, sb, 2, rows), full[rows])


def test_rejects_bad_granularity(orc):
    a = np.zeros((1, 128), np.uint8)
    with pytest.raises(AssertionError):
        orc.gemm_rows(a, np.ones(1, np.float32), 2, a, np.ones(1, np.float32), 0, [0])
