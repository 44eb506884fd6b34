"""GPU parity for fp8_quantize_many (several tensors, one launch) against the oracle.

Every entry must produce exactly the codes and scales the oracle gives for its own granularity
(bit-exact; NaN codes as a class), and the same bytes as separate fp8_quantize calls: mixed
granularities, ragged rows and columns, empty entries, eight entries, both formats, special
values, and the configuration-1 pair (the 14336x4096 weight in 128x128 blocks with the 8192x4096
activations in 1x128 groups) at full size.
"""
import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import assert_codes_equal, assert_f32_bits_equal, dev_bf16, host

pytestmark = pytest.mark.gpu

GR = {1: "GROUP_1x128", 2: "BLOCK_128x128"}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fq.lib()
    assert fq.device_status() == 0
    yield
    assert fq.device_status() == 0, "a kernel's bounded wait gave up"


def check_many(orc, tensors, fmt):
    """tensors: list of (bf16 bits array, granularity)."""
    out = fq.fp8_quantize_many([(dev_bf16(x), g) for x, g in tensors], fmt)
    torch.cuda.synchronize()
    for (x, g), (c, s) in zip(tensors, out):
        oc, os_ = orc.quantize(x, fmt, g)
        assert_codes_equal(host(c), oc, fmt, f"codes {x.shape} {GR[g]}")
        assert_f32_bits_equal(host(s), os_, f"scales {x.shape} {GR[g]}")
    return out


@pytest.mark.parametrize("fmt", [0, 1])
def test_weight_and_activations(orc, fmt):
    w = synth.weight_8b(seed=1, n=384, k=640)
    x = synth.activations(seed=1, m=300, k=640)
    check_many(orc, [(w, 2), (x, 1)], fmt)


@pytest.mark.parametrize("fmt", [0, 1])
def test_ragged_and_empty(orc, fmt):
    tensors = [(synth.activations(seed=2, m=129, k=136), 1), (synth.weight_8b(seed=2, n=200, k=264), 2),
               (np.zeros((0, 128), np.uint16), 1), (synth.activations(seed=3, m=1, k=8), 2),
               (synth.weight_8b(seed=3, n=127, k=1000), 2)]
    check_many(orc, tensors, fmt)


def test_eight_tensors_match_separate_calls(orc):
    tensors = [(synth.activations(seed=10 + j, m=64 + 37 * j, k=128 * (1 + j % 3) + 8 * j), 1 + j % 2)
               for j in range(8)]
    out = check_many(orc, tensors, 0)
    for (x, g), (c, s) in zip(tensors, out):
        c2, s2 = fq.fp8_quantize(dev_bf16(x), fq.E4M3, g)
        torch.cuda.synchronize()
        assert np.array_equal(host(c), host(c2)) and np.array_equal(host(s).view(np.uint32), host(s2).view(np.uint32))


def test_special_values(orc):
    x = synth.per_tensor_1024(seed=4, rows=256, cols=256).copy()
    x[0, :128] = 0                                   # an all-zero group and block row
    x[5, 3] = 0x7FC0                                 # NaN
    x[130, 200] = 0x7F80                             # +Inf
    x[200, 17] = 0x0001                              # subnormal
    check_many(orc, [(x, 1), (x, 2)], 0)


def test_config1_pair_full_size(orc):
    w = synth.weight_8b(seed=1)
    x = synth.activations(seed=1)
    check_many(orc, [(w, 2), (x, 1)], 0)
