"""GPU parity for the block-scaled FP8 GEMM against the oracle's fp64 product.

Operands are quantized by the oracle on the CPU and the same codes and scales go to both
sides.  Tolerance (bf16 output vs the fp64 product of the dequantized operands):
relative Frobenius error <= 5e-3 and every element within 1e-2 * max(|ref|, 1e-2).
Small shapes cover partial M tiles, N not a multiple of the 256-column tile and every scale
combination; the configuration shapes are checked on sampled rows (one per 128-row M tile at
varying offsets, plus the first and last row), which touch every output tile.
"""
import time

import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import dev, host

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
    bound = ELEM * np.maximum(np.abs(ref), 1e-2)
    bad = np.abs(got - ref) > bound
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e}"
    assert not bad.any(), f"{what}: {bad.sum()} elements out of bound, e.g. got {got[bad][:4]} ref {ref[bad][:4]}"
    return rel


def operands(orc, M, N, K, ga, gb, seed, x=None, w=None):
    if x is None:
        x = synth.activations(seed=seed, m=M, k=K)
    if w is None:
        w = synth.weight_8b(seed=seed, n=N, k=K)
    a, sa = orc.quantize(x, orc.E4M3, orc.GROUP_1x128 if ga == 1 else orc.PER_TENSOR)
    b, sb = orc.quantize(w, orc.E4M3, orc.BLOCK_128x128 if gb == 2 else orc.PER_TENSOR)
    return a, sa, b, sb


def run_gpu(a, sa, b, sb, ga, gb):
    c = fq.fp8_gemm_blockscaled(dev(a), dev(sa), dev(b), dev(sb), ga, gb)
    torch.cuda.synchronize()
    return host(c)


def sample_rows(M, seed=0):
    rng = np.random.default_rng(seed)
    rows = [0, M - 1] + [t * 128 + int(rng.integers(0, min(128, M - t * 128))) for t in range((M + 127) // 128)]
    return np.unique(np.array(rows, np.int64))


@pytest.mark.parametrize("ga,gb", [(1, 2), (0, 0), (1, 0), (0, 2)])
@pytest.mark.parametrize("shape", [(1, 128, 128), (16, 256, 256), (128, 256, 128), (130, 384, 512),
                                   (300, 512, 384), (257, 128, 1024)])
def test_gemm_small(orc, ga, gb, shape):
    M, N, K = shape
    a, sa, b, sb = operands(orc, M, N, K, ga, gb, seed=M + N + K)
    got = run_gpu(a, sa, b, sb, ga, gb)
    ref = orc.gemm_rows(a, sa, ga, b, sb, gb, np.arange(M))
    check_tolerance(got, ref, f"{shape} gA={ga} gB={gb}")


def test_gemm_exact_small_integers(orc):
    """Codes of small integers with unit scales: fp32 accumulation is exact, the output is the
    integer product rounded once to bf16."""
    rng = np.random.default_rng(3)
    M, N, K = 64, 256, 256
    vals = np.array([0.0, 1.0, -1.0, 2.0, -2.0, 3.0, -4.0], np.float32)
    A = orc.encode(vals[rng.integers(0, vals.size, (M, K))], orc.E4M3)
    B = orc.encode(vals[rng.integers(0, vals.size, (N, K))], orc.E4M3)
    one = np.ones(1, np.float32)
    got = run_gpu(A, one, B, one, fq.PER_TENSOR, fq.PER_TENSOR)
    ref = orc.gemm_rows(A, one, 0, B, one, 0, np.arange(M))
    want = (ref.astype(np.float32).view(np.uint32) + 0x7FFF + ((ref.astype(np.float32).view(np.uint32) >> 16) & 1)) >> 16
    assert np.array_equal(got.astype(np.uint32), want)


def test_gemm_block_scale_selection(orc):
    """A single nonzero K block: the output must carry exactly that block's scales."""
    M, N, K = 128, 256, 512
    A = np.zeros((M, K), np.uint8)
    B = np.zeros((N, K), np.uint8)
    A[:, 256:384] = 0x38      # 1.0 in K block 2
    B[:, 256:384] = 0x38
    sa = (np.arange(4 * M, dtype=np.float32).reshape(4, M) % 7 + 1) / 8
    sb = (np.arange(2 * 4, dtype=np.float32).reshape(2, 4) + 1) / 4
    got = run_gpu(A, sa, B, sb, fq.GROUP_1x128, fq.BLOCK_128x128)
    ref = orc.gemm_rows(A, sa, 1, B, sb, 2, np.arange(M))
    check_tolerance(got, ref, "single block")


@pytest.mark.parametrize("ga,gb", [(1, 2), (0, 0)])
@pytest.mark.parametrize("M", [1, 7, 16, 33, 48, 57, 64, 65])
@pytest.mark.parametrize("NK", [(128, 128), (384, 640), (1024, 4096), (2048, 1280)])
def test_gemm_decode_split(orc, ga, gb, M, NK):
    """Decode shapes (M <= 64) split the (weight tile, K block) units over all SMs; these N, K
    give ranges that start and end inside tiles, a tile spread over several CTAs and a single
    unit.  M rounds up to 16, 48 or 64 tokens on the MMA's N side (57: zero-filled rows on the
    64-token path, whose scale products come from the scale warp); M = 65 is the first shape past
    the split path."""
    N, K = NK
    a, sa, b, sb = operands(orc, M, N, K, ga, gb, seed=7 * M + N + K)
    got = run_gpu(a, sa, b, sb, ga, gb)
    ref = orc.gemm_rows(a, sa, ga, b, sb, gb, np.arange(M))
    check_tolerance(got, ref, f"M={M} N={N} K={K} gA={ga} gB={gb}")


def test_gemm_decode_deterministic(orc):
    """The split path adds a tile's partial sums in a fixed order: two runs agree bit for bit."""
    M, N, K = 16, 2048, 4096
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, seed=11)
    args = (dev(a), dev(sa), dev(b), dev(sb), 1, 2)
    first = fq.fp8_gemm_blockscaled(*args)
    second = fq.fp8_gemm_blockscaled(*args)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), second.view(torch.int16))


def test_gemm_decode_workspace_left_zero(orc):
    """A caller-provided zero-filled workspace: the per-tile counters are zero again afterwards,
    so the same workspace serves the next call."""
    M, N, K = 16, 2048, 4096
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, seed=12)
    ws = torch.zeros(fq.gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    args = (dev(a), dev(sa), dev(b), dev(sb), 1, 2)
    ref = orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M))
    for _ in range(3):
        got = fq.fp8_gemm_blockscaled(*args, ws=ws)
        torch.cuda.synchronize()
        check_tolerance(host(got), ref, "reused workspace")
        assert int(ws[: 4 * (N // 128)].count_nonzero()) == 0
    assert fq.device_status() == 0


def test_gemm_decode_workspace_reused_across_shapes(orc):
    """One zero-filled workspace serves decode calls of different shapes in turn: after each call
    its counter region (the first 64 KB) is zero again; the partial slots behind it are scratch."""
    shapes = [(16, 1024, 4096), (64, 2048, 1280), (16, 14336, 4096), (33, 384, 640)]
    ws = torch.zeros(max(fq.gemm_workspace_bytes(*s) for s in shapes), dtype=torch.uint8, device="cuda")
    for (M, N, K) in shapes:
        a, sa, b, sb = operands(orc, M, N, K, 1, 2, seed=M * 7 + N)
        got = fq.fp8_gemm_blockscaled(dev(a), dev(sa), dev(b), dev(sb), 1, 2, ws=ws)
        torch.cuda.synchronize()
        assert int(ws[:65536].count_nonzero()) == 0, (M, N, K)
        check_tolerance(host(got), orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M)), f"{M}x{N}x{K}")
    assert fq.device_status() == 0


@pytest.mark.parametrize("M", [16, 64])
def test_gemm_decode_with_sms_taken(orc, M):
    """Forward progress without co-residency: a prefill GEMM with 64 persistent CTAs (each using
    most of an SM's shared memory) holds 64 SMs on one stream while the decode GEMM runs on
    another, so the decode's higher-numbered CTAs can only start once the prefill ends, long after
    the lower ones finished.  Tiles those CTAs share are then completed by whichever CTA counts in
    last.  N = 4096 (32 weight tiles) splits every tile over four to six CTAs.  The output must
    equal the idle-GPU result bit for bit, with no device error and the counters left zero."""
    N, K = 4096, 4096
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, seed=17 + M)
    A, SA, B, SB = dev(a), dev(sa), dev(b), dev(sb)
    ws = torch.zeros(fq.gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    want = fq.fp8_gemm_blockscaled(A, SA, B, SB, 1, 2, ws=ws)
    torch.cuda.synchronize()
    # the hog: 64 M tiles x 1 N tile, K = 131072 (about half a millisecond on 64 SMs)
    ha = torch.zeros((8192, 131072), dtype=torch.uint8, device="cuda")
    hb = torch.zeros((256, 131072), dtype=torch.uint8, device="cuda")
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    hc = torch.empty((8192, 256), dtype=torch.bfloat16, device="cuda")
    s_hog, s_dec = torch.cuda.Stream(), torch.cuda.Stream()
    got = torch.empty_like(want)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for _ in range(3):
        torch.cuda.synchronize()
        with torch.cuda.stream(s_hog):
            ev[0].record(s_hog)
            fq.fp8_gemm_blockscaled(ha, one, hb, one, fq.PER_TENSOR, fq.PER_TENSOR, out=hc)
            ev[1].record(s_hog)
        time.sleep(0.002)                            # the hog's CTAs are resident before the decode starts
        with torch.cuda.stream(s_dec):
            ev[2].record(s_dec)
            fq.fp8_gemm_blockscaled(A, SA, B, SB, 1, 2, out=got, ws=ws)
            ev[3].record(s_dec)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
        assert int(ws[:65536].count_nonzero()) == 0
        print(f"M={M}: hog {ev[0].elapsed_time(ev[1]) * 1e3:.0f} us, decode {ev[2].elapsed_time(ev[3]) * 1e3:.0f} us")
    assert fq.device_status() == 0
    check_tolerance(host(got), orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M)), f"M={M} with SMs taken")


def test_gemm_decode_dirty_workspace_is_reported(orc):
    """Counters at or above a shared tile's number of contributors on entry (here all 0xFF bytes)
    raise device error bit 1: the tile's finishing CTA and its later contributors see the excess at
    once, so the call ends without its bounded wait running out (bit 0 clear); once the workspace
    is zero-filled again the results are right."""
    M, N, K = 16, 2048, 4096
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, seed=13)
    args = (dev(a), dev(sa), dev(b), dev(sb), 1, 2)
    nbytes = fq.gemm_workspace_bytes(M, N, K)
    ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")
    fq.fp8_gemm_blockscaled(*args, ws=ws)
    torch.cuda.synchronize()
    assert fq.device_status() == 2
    ws.zero_()
    got = fq.fp8_gemm_blockscaled(*args, ws=ws)
    torch.cuda.synchronize()
    assert fq.device_status() == 0
    check_tolerance(host(got), orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M)), "after re-zeroing")


def test_gemm_config2_prefill_8b(orc):
    M, N, K = 8192, 14336, 4096
    x = synth.activations(seed=1)
    w = synth.weight_8b(seed=1)
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, 1, x=x, w=w)
    got = run_gpu(a, sa, b, sb, 1, 2)
    rows = sample_rows(M)
    ref = orc.gemm_rows(a, sa, 1, b, sb, 2, rows)
    check_tolerance(got[rows], ref, "config 2 M=8192")


def test_gemm_config2_decode_8b(orc):
    M, N, K = 16, 14336, 4096
    x = synth.activations(seed=1)[:M]
    w = synth.weight_8b(seed=1)
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, 1, x=x, w=w)
    got = run_gpu(a, sa, b, sb, 1, 2)
    ref = orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M))
    check_tolerance(got, ref, "config 2 M=16")


@pytest.mark.parametrize("which", ["up", "down"])
@pytest.mark.parametrize("M", [16384, 64])
def test_gemm_config4_70b(orc, which, M):
    """Prefill: one sampled row in every one of the 128 M tiles (plus the first and last row), so
    every output tile, and every tile of every persistent CTA's walk, is compared."""
    w = synth.weight_70b(seed=4, which=which)
    x = synth.activations_70b(seed=4, m=M, which=which)
    N, K = w.shape
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, 4, x=x, w=w)
    got = run_gpu(a, sa, b, sb, 1, 2)
    rows = sample_rows(M) if M > 64 else np.arange(M)
    assert M <= 64 or np.array_equal(np.unique(rows // 128), np.arange(M // 128))
    ref = orc.gemm_rows(a, sa, 1, b, sb, 2, rows)
    check_tolerance(got[rows], ref, f"config 4 {which} M={M}")


@pytest.mark.parametrize("M", [1024, 16384])
def test_gemm_config4_per_tensor_variant(orc, M):
    """The per-tensor-scale variant at the configuration's prefill size, every M tile sampled."""
    w = synth.weight_70b(seed=4, which="up")
    x = synth.activations_70b(seed=4, m=M, which="up")
    N, K = w.shape
    a, sa, b, sb = operands(orc, M, N, K, 0, 0, 4, x=x, w=w)
    got = run_gpu(a, sa, b, sb, 0, 0)
    rows = sample_rows(M)
    assert np.array_equal(np.unique(rows // 128), np.arange(M // 128))
    ref = orc.gemm_rows(a, sa, 0, b, sb, 0, rows)
    check_tolerance(got[rows], ref, f"config 4 per-tensor M={M}")


# ---------------------------------------------------------------- packed weight tiles

@pytest.mark.parametrize("shape", [(128, 128), (256, 384), (14336, 4096)])
def test_pack_b_tiles_matches_oracle(orc, shape):
    N, K = shape
    b = np.random.default_rng(N + K).integers(0, 256, (N, K)).astype(np.uint8)
    got = fq.fp8_pack_b_tiles(dev(b))
    torch.cuda.synchronize()
    assert np.array_equal(host(got), orc.pack_b_tiles(b))


@pytest.mark.parametrize("ga,gb", [(1, 2), (0, 0)])
@pytest.mark.parametrize("shape", [(1, 128, 128), (16, 256, 256), (64, 384, 512), (130, 384, 512), (300, 512, 384),
                                   (16, 14336, 4096)])
def test_packed_gemm_bit_identical(orc, ga, gb, shape):
    """The packed path feeds the MMAs the same shared-memory bytes: identical bf16 output."""
    M, N, K = shape
    a, sa, b, sb = operands(orc, M, N, K, ga, gb, seed=M + N + K + 7)
    want = run_gpu(a, sa, b, sb, ga, gb)
    bp = fq.fp8_pack_b_tiles(dev(b))
    got = fq.fp8_gemm_blockscaled_packed(dev(a), dev(sa), bp, dev(sb), N, ga, gb)
    torch.cuda.synchronize()
    assert np.array_equal(host(got), want)


def test_packed_gemm_against_oracle(orc):
    M, N, K = 200, 384, 640
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, seed=41)
    got = fq.fp8_gemm_blockscaled_packed(dev(a), dev(sa), dev(orc.pack_b_tiles(b)), dev(sb), N)
    torch.cuda.synchronize()
    check_tolerance(host(got), orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M)), "packed")


# ---------------------------------------------------------------- C quantized in the epilogue

@pytest.mark.parametrize("ga,gb", [(1, 2), (0, 0)])
@pytest.mark.parametrize("shape", [(65, 128, 128), (130, 384, 512), (300, 512, 384), (8192, 14336, 4096)])
def test_gemm_to_fp8_matches_two_steps(orc, ga, gb, shape):
    """Codes and scales equal fp8_gemm_blockscaled followed by fp8_quantize(C, E4M3, 1x128)."""
    M, N, K = shape
    a, sa, b, sb = operands(orc, M, N, K, ga, gb, seed=M + N + K + 3)
    A, SA, B, SB = dev(a), dev(sa), dev(b), dev(sb)
    codes, scales = fq.fp8_gemm_blockscaled_to_fp8(A, SA, B, SB, ga, gb)
    c = fq.fp8_gemm_blockscaled(A, SA, B, SB, ga, gb)
    c2, s2 = fq.fp8_quantize(c, fq.E4M3, fq.GROUP_1x128)
    torch.cuda.synchronize()
    assert np.array_equal(host(codes), host(c2))
    assert np.array_equal(host(scales).view(np.uint32), host(s2).view(np.uint32))


def test_gemm_to_fp8_against_oracle_product(orc):
    """Dequantized output within FP8 rounding (half a step, relative 2^-4) of the fp64 product."""
    M, N, K = 200, 384, 640
    a, sa, b, sb = operands(orc, M, N, K, 1, 2, seed=51)
    codes, scales = fq.fp8_gemm_blockscaled_to_fp8(dev(a), dev(sa), dev(b), dev(sb))
    torch.cuda.synchronize()
    # decoded with torch's float8 type (not the oracle: no CUDA output becomes an oracle input)
    dec = torch.from_numpy(host(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    s_full = np.repeat(host(scales).T, 128, axis=1)[:, :N].astype(np.float64)
    got = dec * s_full
    ref = orc.gemm_rows(a, sa, 1, b, sb, 2, np.arange(M))
    bound = np.abs(ref) * (2.0 ** -4 + 2.0 ** -8 + ELEM) + s_full * 2.0 ** -9 + 1e-2 * 1e-2
    assert np.all(np.abs(got - ref) <= bound)


@pytest.mark.parametrize("ga,gb", [(1, 2), (0, 0)])
def test_gemm_banded_tile_walk_ragged(orc, ga, gb):
    """A (8320 x 8192 codes, 68 MB) above the L2 budget: tiles walk in bands of 16 M tiles, the
    last band is one M tile high (65 tiles) and N = 1408 leaves a half-filled 256-column tile.
    One sampled row per M tile, both scale modes."""
    M, N, K = 8320, 1408, 8192
    assert fq.check_tile_walk(M, N, K) == 0
    a, sa, b, sb = operands(orc, M, N, K, ga, gb, seed=23)
    got = run_gpu(a, sa, b, sb, ga, gb)
    rows = sample_rows(M, seed=23)
    check_tolerance(got[rows], orc.gemm_rows(a, sa, ga, b, sb, gb, rows), f"banded walk gA={ga} gB={gb}")
