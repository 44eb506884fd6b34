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
