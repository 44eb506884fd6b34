"""GPU parity for delayed scaling and the saturation / underflow counts.

A sequence of calls shares one amax history; after every call the codes, the scale bits, the
whole history and the counts must equal the oracle's (bit-exact; NaN codes match as a class).
The tensors change from step to step (different seeds and magnitudes), so later steps cast with
a history that is too small (saturation) or too large (more underflow) for them.
"""
import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import assert_codes_equal, assert_f32_bits_equal, dev, dev_bf16, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fq.lib()
    assert fq.device_status() == 0
    yield
    assert fq.device_status() == 0, "a kernel's bounded wait gave up"


def scaled(x_bits, factor):
    """bf16 bits of x * factor (factor a power of two keeps every value exact)."""
    f = (x_bits.astype(np.uint32) << 16).view(np.float32) * np.float32(factor)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def counts_dev():
    return torch.zeros(2, dtype=torch.int64, device="cuda")


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(1024, 1024), (300, 392), (1, 8)])
def test_per_tensor_sequence(orc, fmt, shape):
    rows, cols = shape
    H = 3
    factors = [1.0, 4.0, 0.25, 16.0, 1.0, 2.0 ** -12]
    h_gpu = torch.zeros(H, dtype=torch.float32, device="cuda")
    h_orc = np.zeros((H, 1), np.float32)
    c_gpu, c_orc = counts_dev(), np.zeros(2, np.uint64)
    for step, f in enumerate(factors):
        x = scaled(synth.per_tensor_1024(seed=step, rows=rows, cols=cols), f)
        codes, scale = fq.fp8_quantize_delayed(dev_bf16(x), h_gpu, step, fmt, counts=c_gpu)
        torch.cuda.synchronize()
        oc, os_ = orc.quantize_delayed(x, fmt, h_orc, step, counts=c_orc)
        assert_f32_bits_equal(host(scale), os_, f"step {step} scale")
        assert_codes_equal(host(codes), oc, fmt, f"step {step} codes")
        assert_f32_bits_equal(host(h_gpu), h_orc[:, 0], f"step {step} history")
        assert host(c_gpu).astype(np.uint64).tolist() == c_orc.tolist(), f"step {step} counts"
    if rows * cols >= 1 << 16:
        assert c_orc[0] > 0 and c_orc[1] > 0     # the sequence exercises both counts


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("gran", [fq.KV_PER_HEAD, fq.KV_PER_TENSOR])
@pytest.mark.parametrize("shape", [(1000, 8, 128), (257, 4, 64), (130, 2, 256)])
def test_kv_sequence(orc, fmt, gran, shape):
    T, Hh, D = shape
    H = 2
    ng = Hh if gran == fq.KV_PER_HEAD else 1
    hk_gpu = torch.zeros((H, ng) if ng > 1 else (H,), dtype=torch.float32, device="cuda")
    hv_gpu = torch.zeros_like(hk_gpu)
    hk, hv = np.zeros((H, ng), np.float32), np.zeros((H, ng), np.float32)
    c_gpu, c_orc = counts_dev(), np.zeros(2, np.uint64)
    for step, f in enumerate([1.0, 8.0, 0.5, 1.0]):
        k, v = synth.kv_70b(seed=10 + step, tokens=T, heads=Hh, head_dim=D)
        k, v = scaled(k, f), scaled(v, 1.0 / f)
        kc, vc, ks, vs = fq.fp8_kv_quantize_delayed(dev_bf16(k), dev_bf16(v), hk_gpu, hv_gpu, step, fmt, gran,
                                                    counts=c_gpu)
        torch.cuda.synchronize()
        okc, oks = orc.quantize_delayed(k, fmt, hk, step, counts=c_orc)
        ovc, ovs = orc.quantize_delayed(v, fmt, hv, step, counts=c_orc)
        assert_f32_bits_equal(host(ks).reshape(-1), oks, f"step {step} k scales")
        assert_f32_bits_equal(host(vs).reshape(-1), ovs, f"step {step} v scales")
        assert_codes_equal(host(kc), okc, fmt, f"step {step} k codes")
        assert_codes_equal(host(vc), ovc, fmt, f"step {step} v codes")
        assert_f32_bits_equal(host(hk_gpu).reshape(H, ng), hk, f"step {step} k history")
        assert_f32_bits_equal(host(hv_gpu).reshape(H, ng), hv, f"step {step} v history")
        assert host(c_gpu).astype(np.uint64).tolist() == c_orc.tolist(), f"step {step} counts"


def test_zero_and_nan_history(orc):
    x = synth.per_tensor_1024(seed=3, rows=64, cols=256)
    for hist in (np.zeros(4, np.float32), np.array([1.0, np.nan, 0.0, 2.0], np.float32)):
        h_gpu, h_orc = dev(hist.copy()), hist.copy().reshape(4, 1)
        c_gpu, c_orc = counts_dev(), np.zeros(2, np.uint64)
        codes, scale = fq.fp8_quantize_delayed(dev_bf16(x), h_gpu, 5, 0, counts=c_gpu)
        torch.cuda.synchronize()
        oc, os_ = orc.quantize_delayed(x, 0, h_orc, 5, counts=c_orc)
        assert_f32_bits_equal(host(scale), os_)
        assert_codes_equal(host(codes), oc, 0)
        assert_f32_bits_equal(host(h_gpu), h_orc[:, 0], "history")
        assert host(c_gpu).astype(np.uint64).tolist() == c_orc.tolist()


def test_empty_tensor_records_zero(orc):
    h = torch.tensor([3.0, 5.0], dtype=torch.float32, device="cuda")
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    _, scale = fq.fp8_quantize_delayed(x, h, 1, 0)
    torch.cuda.synchronize()
    assert host(scale)[0] == np.float32(np.float32(5.0) / np.float32(448.0))
    assert host(h).tolist() == [3.0, 0.0]


def test_step_without_counts_matches(orc):
    """counts = NULL takes the same cast (no counting code) and gives the same codes."""
    x = synth.per_tensor_1024(seed=9, rows=512, cols=512)
    h1 = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    h2 = h1.clone()
    a, sa = fq.fp8_quantize_delayed(dev_bf16(x), h1, 2, 0)
    b, sb = fq.fp8_quantize_delayed(dev_bf16(x), h2, 2, 0, counts=counts_dev())
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(sa, sb) and torch.equal(h1, h2)


def test_kv_config3_full_size_step1(orc):
    """The 70B KV cache of the benchmark configuration: step 0 then one single-pass step."""
    k, v = synth.kv_70b(seed=3)
    kd, vd = dev_bf16(k), dev_bf16(v)
    hk = torch.zeros((2, 8), dtype=torch.float32, device="cuda")
    hv = torch.zeros_like(hk)
    fq.fp8_kv_quantize_delayed(kd, vd, hk, hv, 0, 0, fq.KV_PER_HEAD)
    c_gpu = counts_dev()
    kc, vc, ks, vs = fq.fp8_kv_quantize_delayed(kd, vd, hk, hv, 1, 0, fq.KV_PER_HEAD, counts=c_gpu)
    torch.cuda.synchronize()
    ohk, ohv = np.zeros((2, 8), np.float32), np.zeros((2, 8), np.float32)
    orc.quantize_delayed(k, 0, ohk, 0)
    c_orc = np.zeros(2, np.uint64)
    okc, oks = orc.quantize_delayed(k, 0, ohk, 1, counts=c_orc)
    ovc, ovs = orc.quantize_delayed(v, 0, ohv, 0)
    ovc, ovs = orc.quantize_delayed(v, 0, ohv, 1, counts=c_orc)
    assert_f32_bits_equal(host(ks), oks)
    assert_f32_bits_equal(host(vs), ovs)
    assert_codes_equal(host(kc), okc, 0, "k codes")
    assert_codes_equal(host(vc), ovc, 0, "v codes")
    assert_f32_bits_equal(host(hk), ohk)
    assert host(c_gpu).astype(np.uint64).tolist() == c_orc.tolist()
