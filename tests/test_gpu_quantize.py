"""GPU parity: the CUDA codec, quantizers, dequantizer and KV quantizer against the CPU oracle.

Codes and scales must match bit for bit (a NaN code matches any NaN code of its format).
Sizes: tiny and ragged shapes that span several tiles, every configuration at full size in
the launch configuration the benchmark uses, and two exhaustive sweeps: every fp32 pattern
through the encoder, and every (bf16 x, bf16 amax) pair with |x| <= amax through the fused
1x128 quantizer (the fast reciprocal quotient must equal the IEEE quotient everywhere).
"""
import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import assert_bf16_equal, assert_codes_equal, assert_f32_bits_equal, dev, dev_bf16, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fq.lib()
    assert fq.device_status() == 0
    yield
    assert fq.device_status() == 0, "a kernel's bounded wait gave up"


def quant_gpu(x, fmt, gran):
    c, s = fq.fp8_quantize(dev_bf16(x), fmt, gran)
    torch.cuda.synchronize()
    return host(c), host(s)


def check_quantize(orc, x, fmt, gran):
    c, s = quant_gpu(x, fmt, gran)
    oc, os_ = orc.quantize(x, fmt, gran)
    assert_f32_bits_equal(s, os_)
    assert_codes_equal(c, oc, fmt)
    return c, s


# ------------------------------------------------------------------ codec

@pytest.mark.parametrize("fmt", [0, 1])
def test_decode_all_codes(orc, fmt):
    codes = np.tile(np.arange(256, dtype=np.uint8), 5)[:1001]      # ragged length
    got = host(fq.fp8_decode(dev(codes), fmt))
    want = orc.decode(codes, fmt)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


@pytest.mark.parametrize("fmt", [0, 1])
def test_encode_every_fp32_pattern(orc, fmt):
    chunk = 1 << 28
    for start in range(0, 1 << 32, chunk):
        pats = torch.arange(start, start + chunk, dtype=torch.int64, device="cuda").to(torch.int32).view(torch.float32)
        got = host(fq.fp8_encode(pats, fmt))
        del pats
        want = orc.encode(np.arange(start, start + chunk, dtype=np.uint64).astype(np.uint32).view(np.float32), fmt)
        assert_codes_equal(got, want, fmt, f"encode chunk {start:#x}")


# ------------------------------------------------------------------ quantize: small and ragged

SHAPES = [(1, 8), (1, 128), (3, 136), (4, 1000), (127, 264), (128, 128), (129, 392), (300, 520), (257, 1024)]


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("gran", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES)
def test_quantize_small(orc, fmt, gran, shape):
    rows, cols = shape
    x = synth.activations(seed=rows * 7 + cols, m=rows, k=cols)
    check_quantize(orc, x, fmt, gran)


@pytest.mark.parametrize("gran", [0, 1, 2])
def test_quantize_special_values(orc, gran):
    rows, cols = 130, 392
    x = synth.weight_8b(seed=21, n=rows, k=cols)
    x[0, :] = 0                          # all-zero 1x128 groups
    x[1, :128] = 0x8000                  # negative zeros
    x[2, 5] = 0x0001                     # bf16 subnormals
    x[2, 6] = 0x8003
    x[3, :128] = 0x0002                  # a group of subnormals only (tiny amax -> slow path)
    x[3, 7] = 0x0001
    x[4, 9] = 0x7F7F                     # largest finite bf16
    x[5, 200] = 0x7F80                   # +Inf: the group's scale becomes Inf
    x[6, 300] = 0x7FC0                   # NaN: the group's scale becomes NaN
    for fmt in (0, 1):
        check_quantize(orc, x, fmt, gran)


def test_quantize_empty(orc):
    for gran in (0, 1, 2):
        x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
        c, s = fq.fp8_quantize(x, 0, gran)
        torch.cuda.synchronize()
        assert c.numel() == 0
        if gran == 0:
            assert host(s)[0] == 0.0


# ------------------------------------------------------------------ quantize: exhaustive quotient check

def _pair_rows(a_lo: int, a_hi: int) -> np.ndarray:
    """Rows of 128 bf16 patterns: element 0 is amax pattern a, the other 127 enumerate every
    pattern x in [0, a] (padded with a), with the sign flipped on odd positions."""
    a = np.arange(a_lo, a_hi, dtype=np.int64)
    nrows = (a + 1 + 126) // 127
    row_a = np.repeat(a, nrows)
    first = np.repeat(np.cumsum(nrows) - nrows, nrows)
    j = np.arange(row_a.size) - first
    t = np.arange(127, dtype=np.int64)
    xs = np.minimum(j[:, None] * 127 + t[None, :], row_a[:, None])
    xs = np.where((t % 2 == 1)[None, :], xs | 0x8000, xs)
    return np.concatenate([row_a[:, None], xs], axis=1).astype(np.uint16)


@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_every_x_amax_pair(orc, fmt):
    edges = np.linspace(1, 0x7F80, 17).astype(np.int64)
    for lo, hi in zip(edges[:-1], edges[1:]):
        x = _pair_rows(int(lo), int(hi))
        c, s = quant_gpu(x, fmt, fq.GROUP_1x128)
        oc, os_ = orc.quantize(x, fmt, orc.GROUP_1x128)
        assert_f32_bits_equal(s, os_, f"scales a in [{lo:#x},{hi:#x})")
        assert_codes_equal(c, oc, fmt, f"codes a in [{lo:#x},{hi:#x})")


# ------------------------------------------------------------------ full-size configurations

def test_config0_per_tensor_quant_dequant(orc):
    x = synth.per_tensor_1024(seed=0)
    for fmt in (0, 1):
        c, s = check_quantize(orc, x, fmt, fq.PER_TENSOR)
        y = host(fq.fp8_dequantize(dev(c), dev(s), fmt, fq.PER_TENSOR))
        assert_bf16_equal(y, orc.dequantize(c, s, fmt, orc.PER_TENSOR))


def test_config1_weight_blocks_full(orc):
    w = synth.weight_8b(seed=1)
    check_quantize(orc, w, 0, fq.BLOCK_128x128)


def test_config1_activation_groups_full(orc):
    x = synth.activations(seed=1)
    check_quantize(orc, x, 0, fq.GROUP_1x128)


@pytest.mark.parametrize("gran,fmt", [(fq.KV_PER_HEAD, 0), (fq.KV_PER_HEAD_TOK128, 0), (fq.KV_PER_TENSOR, 1)])
def test_config3_kv_full(orc, gran, fmt):
    k, v = synth.kv_70b(seed=3)
    kc, vc, ks, vs = fq.fp8_kv_quantize(dev_bf16(k), dev_bf16(v), fmt, gran)
    torch.cuda.synchronize()
    okc, ovc, oks, ovs = orc.kv_quantize(k, v, fmt, gran)
    assert_f32_bits_equal(host(ks), oks, "k scales")
    assert_f32_bits_equal(host(vs), ovs, "v scales")
    assert_codes_equal(host(kc), okc, fmt, "k codes")
    assert_codes_equal(host(vc), ovc, fmt, "v codes")


# ------------------------------------------------------------------ KV: small and ragged

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("gran", [0, 1, 2])
@pytest.mark.parametrize("shape", [(1, 1, 8), (5, 3, 16), (130, 2, 128), (257, 8, 64), (300, 4, 256), (129, 1, 136)])
def test_kv_small(orc, fmt, gran, shape):
    T, H, D = shape
    k, v = synth.kv_70b(seed=T + H + D, tokens=T, heads=H, head_dim=D)
    kc, vc, ks, vs = fq.fp8_kv_quantize(dev_bf16(k), dev_bf16(v), fmt, gran)
    torch.cuda.synchronize()
    okc, ovc, oks, ovs = orc.kv_quantize(k, v, fmt, gran)
    assert_f32_bits_equal(host(ks), oks, "k scales")
    assert_f32_bits_equal(host(vs), ovs, "v scales")
    assert_codes_equal(host(kc), okc, fmt, "k codes")
    assert_codes_equal(host(vc), ovc, fmt, "v codes")


# ------------------------------------------------------------------ dequantize

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("gran", [0, 1, 2])
@pytest.mark.parametrize("shape", [(1, 8), (129, 392), (300, 1024)])
def test_dequantize(orc, fmt, gran, shape):
    rows, cols = shape
    x = synth.per_tensor_1024(seed=rows + cols, rows=rows, cols=cols)
    c, s = orc.quantize(x, fmt, gran)
    y = host(fq.fp8_dequantize(dev(c), dev(s), fmt, gran))
    assert_bf16_equal(y, orc.dequantize(c, s, fmt, gran))


@pytest.mark.parametrize("fmt", [0, 1])
def test_dequantize_every_code(orc, fmt):
    c = np.tile(np.arange(256, dtype=np.uint8), 64).reshape(128, 128)
    s = np.array([1.0, 0.37, 3.0e-5, 2.5e30], np.float32)
    for sv in s:
        sc = np.array([sv], np.float32)
        y = host(fq.fp8_dequantize(dev(c), dev(sc), fmt, fq.PER_TENSOR))
        assert_bf16_equal(y, orc.dequantize(c, sc, fmt, orc.PER_TENSOR))
