"""Failure detection on the GPU, tested without a fault.

A self-test kernel waits, through the library's own bounded wait, on a barrier that nothing
ever completes.  The wait must give up after its limit, record bit 0 in the device status, and
return: the status reads 1, reading it clears it, and the context keeps working (a quantization
afterwards matches the oracle bit for bit).  No trap, no bad address, no endless loop.
"""
import time

import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import dev_bf16, host

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable(orc):
    assert torch.cuda.is_available()
    fq.lib()
    assert fq.device_status() == 0
    t0 = time.time()
    fq.selftest_wait_timeout()
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert 1.5 < elapsed < 30, f"the wait should give up after its ~2 s limit, took {elapsed:.1f} s"
    assert fq.device_status() == 1          # bit 0: a bounded wait gave up
    assert fq.device_status() == 0          # reading cleared it
    x = synth.activations(seed=5, m=64, k=256)
    c, s = fq.fp8_quantize(dev_bf16(x), fq.E4M3, fq.GROUP_1x128)
    torch.cuda.synchronize()
    oc, os_ = orc.quantize(x, orc.E4M3, orc.GROUP_1x128)
    assert np.array_equal(host(c), oc) and np.array_equal(host(s).view(np.uint32), os_.view(np.uint32))
    assert fq.device_status() == 0
