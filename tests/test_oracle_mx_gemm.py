"""Pins for the oracle's MXFP8 GEMM and the blocked scale layout (CPU only).

The product (api.makesence.top "LLM推理量化:FP8 versus INT8", the Microscaling passage: one
power-of-two scale per 32 consecutive elements; wangyu.me "大语言模型量化技术（五）：FP8",
"FP8 矩阵乘": FP8 products accumulated in high precision, the scales multiplied back):
    C[m][n] = sum_k decode(A[m][k]) 2^(sA[m][k/32]-127) * decode(B[n][k]) 2^(sB[n][k/32]-127).

Pins, none of which retypes that sum:
  * uniform scale bytes reduce it to a plain matmul of decoded codes (numpy, with torch's float8
    decode), times 2^(ka + kb); mixed formats (A E4M3, B E5M2) catch a swapped format;
  * codes nonzero in one 32-column group only: the other groups' scales drop out, and the result
    divided by that group's two scales is the slice's plain matmul, for every group position
    (catches a group index of k/128, k%32 or a transposed scale array);
  * raising every scale byte of one row (one column) by one doubles exactly that row (column);
  * a NaN scale byte (255) turns exactly its row into NaN;
  * hand-worked byte positions of the blocked layout, and that it is a permutation;
  * hand-worked byte positions of the packed B tile layout (the GEMM's bulk-copy weight format),
    and that each packed row is its tile row with the 16-byte pieces XOR-permuted by row % 8.
"""
import numpy as np
import pytest
import torch

TORCH = {0: torch.float8_e4m3fn, 1: torch.float8_e5m2}


def dec(codes, fmt):
    """Library decode: torch's float8 types, exact in fp64."""
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(TORCH[fmt])
    return t.to(torch.float64).numpy()


def finite_codes(rng, shape, fmt):
    """Random finite codes (no NaN; E5M2 also no Inf)."""
    c = rng.integers(0, 256, shape).astype(np.uint8)
    bad = (c & 0x7F) == 0x7F if fmt == 0 else (c & 0x7C) == 0x7C
    c[bad] &= 0xF0 if fmt == 0 else 0xF3
    return c


@pytest.mark.parametrize("fa,fb", [(0, 0), (1, 1), (0, 1)])
def test_uniform_scales_reduce_to_matmul(orc, fa, fb):
    rng = np.random.default_rng(11 + fa + 2 * fb)
    M, N, K = 37, 45, 160
    A, B = finite_codes(rng, (M, K), fa), finite_codes(rng, (N, K), fb)
    ka, kb = -3, 5
    sa = np.full((M, K // 32), 127 + ka, np.uint8)
    sb = np.full((N, K // 32), 127 + kb, np.uint8)
    got = orc.gemm_mx_rows(A, sa, B, sb, np.arange(M), fa, fb)
    want = (dec(A, fa) @ dec(B, fb).T) * 2.0 ** (ka + kb)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=0)


def test_one_group_special_case(orc):
    rng = np.random.default_rng(12)
    M, N, K = 9, 11, 256
    G = K // 32
    for j in range(G):
        A = np.zeros((M, K), np.uint8)
        A[:, 32 * j:32 * j + 32] = finite_codes(rng, (M, 32), 0)
        B = finite_codes(rng, (N, K), 0)
        sa = rng.integers(100, 150, (M, G)).astype(np.uint8)
        sb = rng.integers(100, 150, (N, G)).astype(np.uint8)
        got = orc.gemm_mx_rows(A, sa, B, sb, np.arange(M))
        # the other groups' scales do not matter
        sa2 = sa.copy()
        sa2[:, [g for g in range(G) if g != j]] += 7
        np.testing.assert_array_equal(orc.gemm_mx_rows(A, sa2, B, sb, np.arange(M)), got)
        slice_mm = dec(A[:, 32 * j:32 * j + 32], 0) @ dec(B[:, 32 * j:32 * j + 32], 0).T
        scale = np.ldexp(1.0, sa[:, j:j + 1].astype(np.int64) - 127) * np.ldexp(1.0, sb[:, j].astype(np.int64) - 127)
        np.testing.assert_allclose(got / scale, slice_mm, rtol=1e-12, atol=0)


def test_row_and_column_doubling(orc):
    rng = np.random.default_rng(13)
    M, N, K = 8, 12, 128
    A, B = finite_codes(rng, (M, K), 0), finite_codes(rng, (N, K), 1)
    sa = rng.integers(110, 140, (M, K // 32)).astype(np.uint8)
    sb = rng.integers(110, 140, (N, K // 32)).astype(np.uint8)
    base = orc.gemm_mx_rows(A, sa, B, sb, np.arange(M), 0, 1)
    sa2 = sa.copy()
    sa2[3] += 1
    got = orc.gemm_mx_rows(A, sa2, B, sb, np.arange(M), 0, 1)
    want = base.copy()
    want[3] *= 2
    np.testing.assert_array_equal(got, want)
    sb2 = sb.copy()
    sb2[5] += 1
    got = orc.gemm_mx_rows(A, sa, B, sb2, np.arange(M), 0, 1)
    want = base.copy()
    want[:, 5] *= 2
    np.testing.assert_array_equal(got, want)


def test_nan_scale_poisons_its_row(orc):
    rng = np.random.default_rng(14)
    M, N, K = 6, 7, 96
    A, B = finite_codes(rng, (M, K), 0), finite_codes(rng, (N, K), 0)
    A[2, 32:64] = 0                                          # zero codes under the NaN scale
    sa = np.full((M, 3), 127, np.uint8)
    sb = np.full((N, 3), 127, np.uint8)
    sa[2, 1] = 255
    got = orc.gemm_mx_rows(A, sa, B, sb, np.arange(M))
    assert np.all(np.isnan(got[2]))
    assert np.all(np.isfinite(np.delete(got, 2, axis=0)))


def test_rows_subset(orc):
    rng = np.random.default_rng(15)
    A, B = finite_codes(rng, (20, 64), 0), finite_codes(rng, (10, 64), 0)
    sa = rng.integers(120, 135, (20, 2)).astype(np.uint8)
    sb = rng.integers(120, 135, (10, 2)).astype(np.uint8)
    full = orc.gemm_mx_rows(A, sa, B, sb, np.arange(20))
    np.testing.assert_array_equal(orc.gemm_mx_rows(A, sa, B, sb, [19, 0, 7]), full[[19, 0, 7]])


def test_blocked_layout_hand_worked(orc):
    rows, ng = 130, 8                                        # two row blocks, two K blocks of 4 groups
    s = np.zeros((rows, ng), np.uint8)
    marks = {(0, 0): 1, (1, 0): 2, (32, 0): 3, (0, 1): 4, (0, 4): 5, (128, 0): 6, (97, 6): 7, (129, 7): 8}
    for (r, j), v in marks.items():
        s[r, j] = v
    b = orc.mx_blocked_scales(s)
    assert b.size == orc.mx_blocked_bytes(rows, ng * 32) == 2 * 2 * 512
    # chunk (row block, K block) at 512 * (rb * 2 + kb); inside, 16 * (r % 32) + 4 * ((r % 128) // 32) + j % 4
    expect = {0: 1, 16: 2, 4: 3, 1: 4, 512: 5, 1024: 6, 512 + 16 * 1 + 4 * 3 + 2: 7, 1536 + 16 * 1 + 3: 8}
    for off, v in expect.items():
        assert b[off] == v, off
    assert np.count_nonzero(b) == len(marks)


def test_blocked_layout_is_a_permutation(orc):
    rows, ng = 256, 8
    s = (np.arange(rows * ng) % 251 + 1).astype(np.uint8).reshape(rows, ng)
    b = orc.mx_blocked_scales(s)
    assert b.size == rows * ng
    np.testing.assert_array_equal(np.sort(b), np.sort(s.ravel()))
    # one chunk holds 128 rows x 4 groups: the first chunk is exactly rows 0..127, groups 0..3
    np.testing.assert_array_equal(np.sort(b[:512]), np.sort(s[:128, :4].ravel()))


def test_packed_b_tiles_hand_worked(orc):
    N, K = 256, 384                                          # 2 x 3 tiles
    b = np.zeros((N, K), np.uint8)
    marks = {(0, 0): 1, (0, 16): 2, (1, 0): 3, (1, 16): 4, (9, 5): 5, (0, 128): 6, (128, 0): 7, (135, 300): 8}
    for (n, k), v in marks.items():
        b[n, k] = v
    p = orc.pack_b_tiles(b)
    assert p.size == N * K
    # tile (nb, kb) at 16384 (3 nb + kb); row r at 128 r; piece j of the row at 16 (j ^ (r % 8))
    expect = {0: 1, 16: 2, 128 + 16: 3, 128 + 0: 4, 9 * 128 + 16 + 5: 5, 16384: 6, 3 * 16384: 7,
              (3 + 2) * 16384 + 7 * 128 + 16 * ((300 - 256) // 16 ^ 7) + (300 % 16): 8}
    for off, v in expect.items():
        assert p[off] == v, off
    assert np.count_nonzero(p) == len(marks)


def test_packed_b_tiles_is_a_permutation_of_whole_tiles(orc):
    rng = np.random.default_rng(31)
    b = rng.integers(0, 256, (256, 256)).astype(np.uint8)
    p = orc.pack_b_tiles(b)
    for nb in range(2):
        for kb in range(2):
            blk = p[(nb * 2 + kb) * 16384:(nb * 2 + kb + 1) * 16384].reshape(128, 128)
            tile = b[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            for r in range(128):                             # each packed row is its tile row, pieces permuted
                assert np.array_equal(np.sort(blk[r]), np.sort(tile[r]))
                assert np.array_equal(blk[r].reshape(8, 16)[np.arange(8) ^ (r % 8)], tile[r].reshape(8, 16))
