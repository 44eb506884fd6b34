"""fp8_kv_quantize_noalloc, the KV quantizer for callers that cannot allocate device memory.

Some callers cannot allocate device memory at all (an engine that reserves all of it up
front, a latency-critical path, a plug-in handed only tensors), so this entry point keeps the
two-pass quantizers' scratch in a fixed array inside the library instead of a caller workspace.
The test calls it through the C ABI twice in a row, on different inputs and granularities, and
checks every output against the regular fp8_kv_quantize bit for bit (the quantizers' parity
bar), so a second call that saw stale scratch from the first would fail.  This file is
collected last; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_quantization_amax_b200 as fq
import synth
from helpers import assert_codes_equal, assert_f32_bits_equal, dev_bf16, host

pytestmark = pytest.mark.gpu


def _call_noalloc(L, k, v, fmt, gran, outs):
    T, H, D = k.shape
    kc, vc, ks, vs = outs
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = L.fp8_kv_quantize_noalloc(p(k), p(v), T, H, D, fmt, gran, p(kc), p(vc), p(ks), p(vs),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _outputs(k, gran):
    T, H, D = k.shape
    shp = fq.kv_scale_shape(T, H, gran)
    return (torch.empty(k.shape, dtype=torch.uint8, device="cuda"), torch.empty(k.shape, dtype=torch.uint8, device="cuda"),
            torch.empty(shp, dtype=torch.float32, device="cuda"), torch.empty(shp, dtype=torch.float32, device="cuda"))


def test_noalloc_matches_workspace_entry_point_twice():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    L = fq.lib()
    assert fq.device_status() == 0
    cases = [((4096, 8, 128), 3, fq.KV_PER_HEAD, fq.E4M3),      # first call: per-head E4M3
             ((3000, 8, 128), 5, fq.KV_PER_TENSOR, fq.E5M2),     # second call: other data, per-tensor E5M2
             ((1000, 8, 128), 7, fq.KV_PER_HEAD_TOK128, fq.E4M3)]  # one-pass granularity: no scratch used
    for shape, seed, gran, fmt in cases:
        T, H, D = shape
        k_np, v_np = synth.kv_70b(seed=seed, tokens=T, heads=H, head_dim=D)
        k, v = dev_bf16(k_np), dev_bf16(v_np)
        outs = _outputs(k, gran)
        assert _call_noalloc(L, k, v, fmt, gran, outs) == 0
        ref = fq.fp8_kv_quantize(k, v, fmt, gran)
        torch.cuda.synchronize()
        got = [host(t) for t in outs]
        want = [host(t) for t in ref]
        assert_codes_equal(got[0], want[0], fmt, "k codes")
        assert_codes_equal(got[1], want[1], fmt, "v codes")
        assert_f32_bits_equal(got[2], want[2], "k scales")
        assert_f32_bits_equal(got[3], want[3], "v scales")
    assert fq.device_status() == 0


def test_noalloc_refuses_more_heads_than_its_scratch_holds():
    L = fq.lib()
    k = torch.zeros((16, 64, 8), dtype=torch.bfloat16, device="cuda")
    outs = _outputs(k, fq.KV_PER_HEAD)
    assert _call_noalloc(L, k, k, fq.E4M3, fq.KV_PER_HEAD, outs) == 3     # FP8Q_ERR_WORKSPACE
