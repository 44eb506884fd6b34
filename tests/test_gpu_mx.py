"""GPU parity for the MXFP8 quantizer and dequantizer against the oracle (bit-exact).

Codes and byte exponents must equal the oracle's (NaN codes match as a class); dequantized
bf16 must be bit-identical.  Shapes include ragged column counts (a partial 128-column box),
the configuration-1 activations at full size, and special groups (all zero, subnormal amax,
amax near the bf16 maximum, NaN, Inf).
"""
import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import assert_bf16_equal, assert_codes_equal, dev, dev_bf16, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fq.lib()
    assert fq.device_status() == 0
    yield
    assert fq.device_status() == 0, "a kernel's bounded wait gave up"


def check(orc, x, fmt):
    codes, scales = fq.fp8_quantize_mx(dev_bf16(x), fmt)
    torch.cuda.synchronize()
    oc, os_ = orc.quantize_mx(x, fmt)
    assert np.array_equal(host(scales), os_), "scale exponents differ"
    assert_codes_equal(host(codes), oc, fmt)
    return oc, os_


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(1, 32), (64, 128), (129, 416), (300, 1024), (3, 4096)])
def test_quantize_mx(orc, fmt, shape):
    rows, cols = shape
    check(orc, synth.activations(seed=rows + cols, m=rows, k=cols), fmt)


@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_mx_config1_full(orc, fmt):
    check(orc, synth.activations(seed=1), fmt)


@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_mx_special_groups(orc, fmt):
    x = synth.per_tensor_1024(seed=4, rows=8, cols=256).copy()
    bits = lambda v: (np.float32(v).view(np.uint32) >> 16).astype(np.uint16)  # noqa: E731 (exact values only)
    x[0, :32] = 0                                         # all-zero group
    x[1, 32:64] = bits(2.0 ** -133)                       # subnormal amax: clamped exponent
    x[2, 64:96] = bits(3.3895313892515355e38)             # near the bf16 maximum
    x[2, 70] = 0xFF7F                                     # -max
    x[3, 96:128] = bits(448.0)                            # exactly FMAX (E4M3): k = 0
    x[3, 128] = bits(450.0)                               # just above
    x[4, 160] = 0x7FC0                                    # NaN
    x[5, 192] = 0x7F80                                    # +Inf
    x[6, 224:256] = bits(2.0 ** -126)                     # smallest normal
    check(orc, x, fmt)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(1, 32), (129, 416), (1024, 1024)])
def test_dequantize_mx(orc, fmt, shape):
    rows, cols = shape
    rng = np.random.default_rng(rows + cols + fmt)
    codes = rng.integers(0, 256, (rows, cols)).astype(np.uint8)
    scales = rng.integers(90, 165, (rows, cols // 32)).astype(np.uint8)
    scales.flat[::7] = 0
    scales.flat[3::11] = 255
    y = fq.fp8_dequantize_mx(dev(codes), dev(scales), fmt)
    torch.cuda.synchronize()
    assert_bf16_equal(host(y), orc.dequantize_mx(codes, scales, fmt))


def test_mx_roundtrip_error_bound(orc):
    """Dequantized values are within half a grid step (relative 1/16 for E4M3) of the input."""
    x = synth.activations(seed=6, m=256, k=1024)
    codes, scales = fq.fp8_quantize_mx(dev_bf16(x), 0)
    y = host(fq.fp8_dequantize_mx(codes, scales, 0))
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    yf = (y.astype(np.uint32) << 16).view(np.float32)
    k = np.repeat(host(scales).astype(np.int32) - 127, 32, axis=1)
    tiny = np.ldexp(1.0, k - 9)                           # the least subnormal step at this scale
    assert np.all(np.abs(yf - xf) <= np.maximum(np.abs(xf) / 16 * 1.04, tiny))
