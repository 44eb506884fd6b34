"""GPU parity for the scale-health counts against the oracle (exact counts).

The scale histogram runs on real scale arrays (1x128 and 128x128 quantization, the KV cache's
per-head x 128-token scales, MXFP8 bytes) and on hand-made arrays with zero, subnormal, NaN and
Inf scales; the underflow count on the codes of a quantization whose small values flush to
zero, including lengths that are not a multiple of the kernel's eight-element vectors.

No CUDA output becomes an oracle input: the expected histogram and count come from the
oracle's own quantization of the same input.  Each case checks the counting kernel on the
oracle's scales or codes, and then the whole GPU chain (the GPU's quantizer followed by its
counting kernel) against the same expected value.
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
    assert fq.device_status() == 0


def gpu_hist(scales_t):
    h = fq.fp8_scale_histogram(scales_t)
    torch.cuda.synchronize()
    return host(h).astype(np.uint32)


@pytest.mark.parametrize("gran", [fq.GROUP_1x128, fq.BLOCK_128x128])
def test_histogram_of_quantizer_scales(orc, gran):
    x = synth.activations(seed=3, m=1000, k=2048)
    _, want_s = orc.quantize(x, orc.E4M3, gran)
    want = orc.scale_histogram(want_s)
    assert np.array_equal(gpu_hist(dev(want_s)), want)
    _, s = fq.fp8_quantize(dev_bf16(x), fq.E4M3, gran)
    assert np.array_equal(gpu_hist(s), want)


def test_histogram_of_kv_scales(orc):
    k, v = synth.kv_70b(seed=3, tokens=4096)
    want_ks = orc.kv_quantize(k, v, orc.E4M3, fq.KV_PER_HEAD_TOK128)[2]
    want = orc.scale_histogram(want_ks)
    assert np.array_equal(gpu_hist(dev(want_ks)), want)
    ks = fq.fp8_kv_quantize(dev_bf16(k), dev_bf16(v), fq.E4M3, fq.KV_PER_HEAD_TOK128)[2]
    assert np.array_equal(gpu_hist(ks), want)


def test_histogram_of_mx_bytes(orc):
    x = synth.activations(seed=1)
    _, want_s = orc.quantize_mx(x, orc.E4M3)
    want = orc.scale_histogram(want_s)
    assert np.array_equal(gpu_hist(dev(want_s)), want)
    _, s = fq.fp8_quantize_mx(dev_bf16(x))
    assert np.array_equal(gpu_hist(s), want)


def test_histogram_special_values_and_accumulation(orc):
    s = np.array([0.0, 1e-40, np.nan, np.inf, -np.inf, 1.0, -1.0, 3.4e38] * 1000 + [448.0] * 7, np.float32)
    st = dev(s)
    h = fq.fp8_scale_histogram(st)
    fq.fp8_scale_histogram(st, h)                    # a second call adds to the same histogram
    torch.cuda.synchronize()
    assert np.array_equal(host(h).astype(np.uint32), 2 * orc.scale_histogram(s))


@pytest.mark.parametrize("n", [1, 7, 8, 1001, 65543])
def test_underflow_count_small(orc, n):
    rng = np.random.default_rng(n)
    x = rng.integers(0, 1 << 16, n).astype(np.uint16)
    c = rng.integers(0, 256, n).astype(np.uint8)
    c[rng.random(n) < 0.3] = 0x80
    got = fq.fp8_count_underflow(dev_bf16(x), dev(c))
    torch.cuda.synchronize()
    assert int(host(got)[0]) == orc.count_underflow(x, c)


def test_underflow_count_of_a_quantization(orc):
    """Per-tensor scaling of activations with a few large outliers flushes many small values."""
    x = synth.activations(seed=1)
    x = x.copy()
    x[0, :4] = 0x7F00                                # outliers ~1.7e38: every other value underflows
    want_codes, _ = orc.quantize(x, orc.E4M3, orc.PER_TENSOR)
    want = orc.count_underflow(x, want_codes)
    assert want > 1000
    xd = dev_bf16(x)
    from_oracle_codes = fq.fp8_count_underflow(xd, dev(want_codes))
    codes, _ = fq.fp8_quantize(xd, fq.E4M3, fq.PER_TENSOR)
    from_gpu_codes = fq.fp8_count_underflow(xd, codes)
    torch.cuda.synchronize()
    assert int(host(from_oracle_codes)[0]) == want
    assert int(host(from_gpu_codes)[0]) == want
