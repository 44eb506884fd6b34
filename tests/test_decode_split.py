"""Host-side checks (no GPU) of the decode GEMM's work split, through the library's own range
functions (fp8q_check_decode_split): the split-tile hand-off of the decode kernel relies on each
CTA holding at most one segment of a tile a lower CTA started and at most one of a tile it starts
but does not end, on its two warps agreeing which those are, and on every shared tile having one
finishing CTA and each other contributor counted once."""
import itertools

import pytest

import fp8_quantization_amax_b200 as fq

SMS = [1, 2, 3, 7, 37, 100, 132, 148, 160]
NS = [128, 256, 384, 1024, 4096, 8192, 14336, 28672, 57344]
KS = [128, 256, 640, 4096, 8192, 14336, 28672]


@pytest.mark.parametrize("sms", SMS)
def test_decode_split_invariants(sms):
    for M, N, K in itertools.product([1, 16, 64], NS, KS):
        assert fq.check_decode_split(M, N, K, sms) == 0, (M, N, K, sms)


def test_decode_split_model_shapes():
    # the decode shapes of the pages' models on a full B200 (148 SMs) and on partial devices
    for (N, K) in [(14336, 4096), (4096, 14336), (6144, 4096), (57344, 4096), (28672, 8192), (8192, 28672)]:
        for sms in range(1, 149):
            assert fq.check_decode_split(16, N, K, sms) == 0, (N, K, sms)


def test_decode_split_rejects_non_decode_shapes():
    assert fq.check_decode_split(65, 128, 128, 148) == -1
    assert fq.check_decode_split(16, 100, 128, 148) == -1
    assert fq.check_decode_split(16, 128, 100, 148) == -1
    assert fq.check_decode_split(0, 128, 128, 148) == -1
    assert fq.check_decode_split(16, 128, 128, 0) == -1
