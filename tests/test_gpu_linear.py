"""GPU parity for the linear layer with dynamic activation quantization.

fp8_linear_dynamic(X, B) must be bit-identical to fp8_quantize(X, E4M3, 1x128) followed by
fp8_gemm_blockscaled (it issues the same two kernels as dependent launches, with the codes in
its own workspace), and the counters of the GEMM workspace it shares with other calls (its first
64 KB) must stay zero.
Results are also checked against the oracle's fp64 product within the GEMM tolerance.
"""
import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import dev, dev_bf16, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fq.lib()
    assert fq.device_status() == 0
    yield
    assert fq.device_status() == 0, "a kernel's bounded wait gave up"


def two_step(xd, b, sb, gb):
    a, sa = fq.fp8_quantize(xd, fq.E4M3, fq.GROUP_1x128)
    return fq.fp8_gemm_blockscaled(a, sa, b, sb, fq.GROUP_1x128, gb)


def weights(orc, N, K, gb, seed):
    w = synth.weight_8b(seed=seed, n=N, k=K)
    b, sb = orc.quantize(w, orc.E4M3, orc.BLOCK_128x128 if gb == 2 else orc.PER_TENSOR)
    return dev(b), dev(sb)


def assert_same_bits(got, want, what):
    g, w = host(got), host(want)
    bad = np.nonzero(g != w)
    assert bad[0].size == 0, f"{what}: {bad[0].size} elements differ, first at {bad[0][:4]}, {bad[1][:4]}"


@pytest.mark.parametrize("gb", [2, 0])
@pytest.mark.parametrize("shape", [(1, 128, 128), (7, 384, 640), (16, 1024, 4096), (33, 2048, 1280),
                                   (48, 256, 512), (64, 2048, 1280), (65, 384, 512), (300, 512, 384)])
def test_linear_equals_quantize_then_gemm(orc, gb, shape):
    M, N, K = shape
    x = dev_bf16(synth.activations(seed=M + N + K, m=M, k=K))
    b, sb = weights(orc, N, K, gb, seed=N + K)
    got = fq.fp8_linear_dynamic(x, b, sb, gb)
    want = two_step(x, b, sb, gb)
    torch.cuda.synchronize()
    assert_same_bits(got, want, f"{shape} gB={gb}")


def test_linear_special_rows(orc):
    """All-zero rows (amax 0), rows of tiny values (the IEEE slow path), ragged M."""
    M, N, K = 20, 512, 1024
    xs = synth.activations(seed=5, m=M, k=K).copy()
    xs[3] = 0
    xs[4, :128] = 0x8000                                # -0 in one group only
    tiny = np.float32(2.0 ** -70)
    xs[7] = (np.full(K, tiny, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    x = dev_bf16(xs)
    b, sb = weights(orc, N, K, 2, seed=9)
    assert_same_bits(fq.fp8_linear_dynamic(x, b, sb), two_step(x, b, sb, 2), "special rows")


def test_linear_against_oracle(orc):
    M, N, K = 16, 2048, 4096
    xs = synth.activations(seed=21, m=M, k=K)
    b, sb = weights(orc, N, K, 2, seed=22)
    got = host(fq.fp8_linear_dynamic(dev_bf16(xs), b, sb))
    a, sa = orc.quantize(xs, orc.E4M3, orc.GROUP_1x128)
    ref = orc.gemm_rows(a, sa, 1, host(b), host(sb), 2, np.arange(M))
    g = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 5e-3
    assert np.all(np.abs(g - ref) <= 1e-2 * np.maximum(np.abs(ref), 1e-2))


@pytest.mark.parametrize("case", ["8b_m16", "70b_up_m64", "70b_down_m64"])
def test_linear_config_shapes(orc, case):
    if case == "8b_m16":
        w, xs = synth.weight_8b(seed=1), synth.activations(seed=1)[:16]
    else:
        which = case.split("_")[1]
        w, xs = synth.weight_70b(seed=4, which=which), synth.activations_70b(seed=4, m=64, which=which)
    b, sb = orc.quantize(w, orc.E4M3, orc.BLOCK_128x128)
    b, sb, x = dev(b), dev(sb), dev_bf16(xs)
    assert_same_bits(fq.fp8_linear_dynamic(x, b, sb), two_step(x, b, sb, 2), case)


def test_linear_keeps_the_shared_gemm_workspace_zero(orc):
    shapes = [(16, 2048, 4096), (64, 1024, 1280), (7, 384, 640)]
    ws = torch.zeros(max(fq.gemm_workspace_bytes(*s) for s in shapes), dtype=torch.uint8, device="cuda")
    for (M, N, K) in shapes:
        x = dev_bf16(synth.activations(seed=M, m=M, k=K))
        b, sb = weights(orc, N, K, 2, seed=N)
        got = fq.fp8_linear_dynamic(x, b, sb, ws=ws)
        want = two_step(x, b, sb, 2)
        torch.cuda.synchronize()
        assert_same_bits(got, want, f"{M}x{N}x{K}")
        assert int(ws[:65536].count_nonzero()) == 0


# ------------------------------------------------------------------ the fused (one-launch) form

def fused_ws(M, K):
    n = fq.linear_fused_workspace_bytes(M, K)
    return torch.zeros(n, dtype=torch.uint8, device="cuda")


def act_parts(ws, M, K):
    """(codes [M][K], scales [K/128][M]) as the fused kernel's first phase wrote them, after the
    256 bytes of grid-barrier words."""
    n_codes = 256 + (M * K + 255) // 256 * 256
    codes = ws[256:256 + M * K].view(M, K)
    scales = ws[n_codes:n_codes + 4 * (K // 128) * M].view(torch.float32).view(K // 128, M)
    return codes, scales


@pytest.mark.parametrize("gb", [2, 0])
@pytest.mark.parametrize("shape", [(65, 384, 512), (300, 512, 384), (129, 2048, 1280), (1000, 1024, 4096),
                                   (2048, 4096, 4096), (4097, 1536, 2048)])
def test_linear_fused_equals_two_launches(orc, gb, shape):
    """One cooperative launch (quantize phase, grid barrier, GEMM) against the two-launch form:
    the same C bits, and the codes and scales left in act_ws are fp8_quantize's.  Shapes with
    fewer tiles than SMs, several tiles per block (2048 x 4096: 512 tiles) and ragged M."""
    M, N, K = shape
    x = dev_bf16(synth.activations(seed=M + 3 * N + K, m=M, k=K))
    b, sb = weights(orc, N, K, gb, seed=N + K + 1)
    ws = fused_ws(M, K)
    got = fq.fp8_linear_dynamic_fused(x, b, sb, gb, act_ws=ws)
    want = fq.fp8_linear_dynamic(x, b, sb, gb)
    a, sa = fq.fp8_quantize(x, fq.E4M3, fq.GROUP_1x128)
    torch.cuda.synchronize()
    assert_same_bits(got, want, f"{shape} gB={gb}")
    codes, scales = act_parts(ws, M, K)
    assert torch.equal(codes, a), "codes in act_ws differ from fp8_quantize"
    assert torch.equal(scales.view(torch.int32), sa.view(torch.int32)), "scales in act_ws differ"
    assert int(ws[:4].count_nonzero()) == 0, "grid-barrier arrival count not left zero"


def test_linear_fused_special_groups(orc):
    """Groups that take the quantizer's slow path (tiny amax, subnormal bf16, +-inf, NaN), zero
    and -0 groups: the fused phase computes them without a division and must match the
    stand-alone quantizer's IEEE divisions bit for bit."""
    M, N, K = 136, 512, 1024
    xs = synth.activations(seed=6, m=M, k=K).copy()
    xs[3] = 0
    xs[4, :128] = 0x8000
    for r, e in ((7, -70), (8, -100), (9, -126), (10, -61)):
        xs[r] = (np.full(K, np.float32(2.0 ** e), np.float32).view(np.uint32) >> 16).astype(np.uint16)
        xs[r, 1::3] ^= 0x8000
        xs[r, 2::5] = (xs[r, 2::5].astype(np.uint32) - 3).astype(np.uint16)
    xs[11] = np.arange(K, dtype=np.uint16) % 0x80 + 1          # bf16 subnormals only
    xs[12, 5] = 0x7F80                                        # +inf in group 0
    xs[12, 200] = 0xFF80                                      # -inf in group 1
    xs[12, 300] = 0xFF80
    xs[12, 301] = 0x7F80                                      # both infinities in group 2
    xs[13, 17] = 0x7FC0                                       # NaN in group 0
    xs[13, 129] = 0xFFC1                                      # a negative NaN in group 1
    xs[14, 128:256] = 0x7F80                                  # a group of +inf only
    x = dev_bf16(xs)
    b, sb = weights(orc, N, K, 2, seed=10)
    ws = fused_ws(M, K)
    got = fq.fp8_linear_dynamic_fused(x, b, sb, act_ws=ws)
    a, sa = fq.fp8_quantize(x, fq.E4M3, fq.GROUP_1x128)
    want = fq.fp8_gemm_blockscaled(a, sa, b, sb, fq.GROUP_1x128, 2)
    torch.cuda.synchronize()
    codes, scales = act_parts(ws, M, K)
    bad = torch.nonzero(codes != a)
    assert bad.numel() == 0, f"codes differ at {bad[:6].tolist()}"
    assert torch.equal(scales.view(torch.int32), sa.view(torch.int32))
    assert_same_bits(got, want, "special groups")


def test_linear_fused_reuses_its_workspace(orc):
    """One zeroed act_ws serves calls of several shapes in a row (the barrier's arrival count is
    left zero; its generation word counts the calls)."""
    shapes = [(256, 1024, 2048), (65, 384, 512), (1024, 2048, 1280)]
    n = max(fq.linear_fused_workspace_bytes(M, K) for (M, _, K) in shapes)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    for (M, N, K) in shapes * 2:
        x = dev_bf16(synth.activations(seed=M + 1, m=M, k=K))
        b, sb = weights(orc, N, K, 2, seed=N + 2)
        nb = fq.linear_fused_workspace_bytes(M, K)
        got = fq.fp8_linear_dynamic_fused(x, b, sb, act_ws=ws[:nb])
        want = two_step(x, b, sb, 2)
        torch.cuda.synchronize()
        assert_same_bits(got, want, f"{M}x{N}x{K}")
        assert int(ws[:4].count_nonzero()) == 0


def test_linear_fused_against_oracle(orc):
    M, N, K = 200, 1024, 4096
    xs = synth.activations(seed=23, m=M, k=K)
    b, sb = weights(orc, N, K, 2, seed=24)
    got = host(fq.fp8_linear_dynamic_fused(dev_bf16(xs), b, sb))
    a, sa = orc.quantize(xs, orc.E4M3, orc.GROUP_1x128)
    rows = np.arange(0, M, 7)
    ref = orc.gemm_rows(a, sa, 1, host(b), host(sb), 2, rows)
    g = (got[rows].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 5e-3
    assert np.all(np.abs(g - ref) <= 1e-2 * np.maximum(np.abs(ref), 1e-2))


@pytest.mark.parametrize("case", ["8b_m8192", "70b_up_m16384"])
def test_linear_fused_config_shapes(orc, case):
    """The full prefill shapes the benchmark times: bit-identical to the two-launch form."""
    if case == "8b_m8192":
        w, xs = synth.weight_8b(seed=2), synth.activations(seed=2)
    else:
        w, xs = synth.weight_70b(seed=5, which="up"), synth.activations_70b(seed=5, m=16384, which="up")
    b, sb = orc.quantize(w, orc.E4M3, orc.BLOCK_128x128)
    b, sb, x = dev(b), dev(sb), dev_bf16(xs)
    got = fq.fp8_linear_dynamic_fused(x, b, sb)
    want = fq.fp8_linear_dynamic(x, b, sb)
    torch.cuda.synchronize()
    assert_same_bits(got, want, case)


def test_linear_fused_rejects_decode_shapes(orc):
    x = dev_bf16(synth.activations(seed=1, m=64, k=512))
    b, sb = weights(orc, 256, 512, 2, seed=3)
    with pytest.raises(fq.Fp8qError):
        fq.fp8_linear_dynamic_fused(x, b, sb)
