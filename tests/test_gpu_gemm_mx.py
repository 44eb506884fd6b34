"""GPU parity for the MXFP8 GEMM (block-scaled tensor-core MMA) and the blocked-scale quantizer.

The quantizer's codes and blocked scale bytes must equal the oracle's quantize_mx, rearranged by
the oracle's definition of the blocked layout, bit for bit.  The GEMM's bf16 output is compared
with the oracle's fp64 product of the dequantized operands under the block-scaled GEMM's
tolerance: relative Frobenius error <= 5e-3 and every element within 1e-2 * max(|ref|, 1e-2).
Operands come from the oracle's MXFP8 quantizer on seeded synthetic tensors (or from seeded
random codes and scale bytes), the same bytes on both sides.  Shapes cover a single tile, partial
M tiles, N with a half-filled 256-column tile, K of one and of many 128-blocks, every format
pair, and the configuration-2 shape on sampled rows.
"""
import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import assert_codes_equal, dev, dev_bf16, host

pytestmark = pytest.mark.gpu

REL_FRO = 5e-3
ELEM = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fq.lib()
    assert fq.device_status() == 0
    yield
    assert fq.device_status() == 0, "a kernel's bounded wait gave up"


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_tolerance(got_bits, ref, what=""):
    got = bf16_to_f64(got_bits)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    bad = np.abs(got - ref) > ELEM * np.maximum(np.abs(ref), 1e-2)
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e}"
    assert not bad.any(), f"{what}: {bad.sum()} elements out of bound, e.g. got {got[bad][:4]} ref {ref[bad][:4]}"


def sample_rows(M, seed=0):
    rng = np.random.default_rng(seed)
    rows = [0, M - 1] + [t * 128 + int(rng.integers(0, min(128, M - t * 128))) for t in range((M + 127) // 128)]
    return np.unique(np.array(rows, np.int64))


def mx_operands(orc, M, N, K, fa, fb, seed):
    a, sa = orc.quantize_mx(synth.activations(seed=seed, m=M, k=K), fa)
    b, sb = orc.quantize_mx(synth.weight_8b(seed=seed, n=N, k=K), fb)
    return a, sa, b, sb


def run_gpu(orc, a, sa, b, sb, fa, fb):
    c = fq.fp8_gemm_mx(dev(a), dev(orc.mx_blocked_scales(sa)), dev(b), dev(orc.mx_blocked_scales(sb)), fa, fb)
    torch.cuda.synchronize()
    return host(c)


# ---------------------------------------------------------------- blocked-scale quantizer

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(1, 32), (129, 416), (300, 1024), (128, 128), (3, 4096)])
def test_quantize_mx_blocked(orc, fmt, shape):
    rows, cols = shape
    x = synth.activations(seed=rows + cols, m=rows, k=cols)
    codes, scales = fq.fp8_quantize_mx_blocked(dev_bf16(x), fmt)
    torch.cuda.synchronize()
    oc, os_ = orc.quantize_mx(x, fmt)
    assert_codes_equal(host(codes), oc, fmt)
    assert np.array_equal(host(scales), orc.mx_blocked_scales(os_)), "blocked scale bytes differ"


def test_quantize_mx_blocked_config1_full(orc):
    x = synth.activations(seed=1)
    codes, scales = fq.fp8_quantize_mx_blocked(dev_bf16(x), 0)
    torch.cuda.synchronize()
    oc, os_ = orc.quantize_mx(x, 0)
    assert_codes_equal(host(codes), oc, 0)
    assert np.array_equal(host(scales), orc.mx_blocked_scales(os_))


# ---------------------------------------------------------------- GEMM

@pytest.mark.parametrize("fa,fb", [(0, 0), (1, 1), (0, 1), (1, 0)])
@pytest.mark.parametrize("shape", [(128, 256, 128), (1, 128, 128), (130, 384, 512), (300, 512, 384),
                                   (257, 128, 1024)])
def test_gemm_mx_small(orc, fa, fb, shape):
    M, N, K = shape
    a, sa, b, sb = mx_operands(orc, M, N, K, fa, fb, seed=M + N + K)
    got = run_gpu(orc, a, sa, b, sb, fa, fb)
    check_tolerance(got, orc.gemm_mx_rows(a, sa, b, sb, np.arange(M), fa, fb), f"{shape} fa={fa} fb={fb}")


def test_gemm_mx_random_codes_and_exponents(orc):
    """Every finite code and per-group exponents spread over 2^-8 .. 2^8 on each side."""
    rng = np.random.default_rng(21)
    M, N, K = 200, 384, 640
    a = rng.integers(0, 256, (M, K)).astype(np.uint8)
    b = rng.integers(0, 256, (N, K)).astype(np.uint8)
    a[(a & 0x7F) == 0x7F] &= 0xF0                        # E4M3 NaN codes -> finite
    b[(b & 0x7F) == 0x7F] &= 0xF0
    sa = rng.integers(119, 136, (M, K // 32)).astype(np.uint8)
    sb = rng.integers(119, 136, (N, K // 32)).astype(np.uint8)
    got = run_gpu(orc, a, sa, b, sb, 0, 0)
    check_tolerance(got, orc.gemm_mx_rows(a, sa, b, sb, np.arange(M)), "random codes")


def test_gemm_mx_group_locality(orc):
    """Codes nonzero in one 32-column group per K block: each output comes from one scale pair."""
    rng = np.random.default_rng(22)
    M, N, K = 128, 256, 512
    a = np.zeros((M, K), np.uint8)
    for kb in range(K // 128):
        j = kb % 4
        a[:, kb * 128 + 32 * j: kb * 128 + 32 * j + 32] = rng.integers(0, 0x7E, (M, 32)).astype(np.uint8)
    b = rng.integers(0, 0x7E, (N, K)).astype(np.uint8)
    sa = rng.integers(110, 145, (M, K // 32)).astype(np.uint8)
    sb = rng.integers(110, 145, (N, K // 32)).astype(np.uint8)
    got = run_gpu(orc, a, sa, b, sb, 0, 0)
    check_tolerance(got, orc.gemm_mx_rows(a, sa, b, sb, np.arange(M)), "group locality")


def test_gemm_mx_quantizer_chain(orc):
    """GPU quantizer (blocked scales) straight into the GPU GEMM, against the oracle chain."""
    M, N, K = 256, 512, 1024
    x = synth.activations(seed=23, m=M, k=K)
    w = synth.weight_8b(seed=23, n=N, k=K)
    ca, sa = fq.fp8_quantize_mx_blocked(dev_bf16(x), 0)
    cb, sb = fq.fp8_quantize_mx_blocked(dev_bf16(w), 0)
    c = fq.fp8_gemm_mx(ca, sa, cb, sb)
    torch.cuda.synchronize()
    a, osa = orc.quantize_mx(x, 0)
    b, osb = orc.quantize_mx(w, 0)
    check_tolerance(host(c), orc.gemm_mx_rows(a, osa, b, osb, np.arange(M)), "chain")


def test_gemm_mx_deterministic(orc):
    M, N, K = 300, 512, 1024
    a, sa, b, sb = mx_operands(orc, M, N, K, 0, 0, seed=24)
    args = (dev(a), dev(orc.mx_blocked_scales(sa)), dev(b), dev(orc.mx_blocked_scales(sb)))
    c1 = host(fq.fp8_gemm_mx(*args))
    c2 = host(fq.fp8_gemm_mx(*args))
    assert np.array_equal(c1, c2)


@pytest.mark.parametrize("M", [16, 8192])
def test_gemm_mx_config2_sampled(orc, M):
    N, K = 14336, 4096
    x = synth.activations(seed=2, m=M, k=K)
    w = synth.weight_8b(seed=2, n=N, k=K)
    a, sa = orc.quantize_mx(x, 0)
    b, sb = orc.quantize_mx(w, 0)
    got = run_gpu(orc, a, sa, b, sb, 0, 0)
    rows = sample_rows(M, seed=M)
    check_tolerance(got[rows], orc.gemm_mx_rows(a, sa, b, sb, rows), f"M={M} sampled")


def test_gemm_mx_banded_tile_walk(orc):
    """A (8192 x 8192 codes, 64 MB) above the L2 budget, so tiles walk in bands of 16 M tiles;
    N = 1280 leaves a half-filled 256-column tile in every band.  One sampled row per M tile."""
    M, N, K = 8192, 1280, 8192
    assert fq.check_tile_walk(M, N, K) == 0
    a, sa = orc.quantize_mx(synth.activations(seed=9, m=M, k=K), 0)
    b, sb = orc.quantize_mx(synth.weight_8b(seed=9, n=N, k=K), 0)
    got = run_gpu(orc, a, sa, b, sb, 0, 0)
    rows = sample_rows(M, seed=9)
    check_tolerance(got[rows], orc.gemm_mx_rows(a, sa, b, sb, rows), "banded walk")
