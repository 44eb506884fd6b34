"""Host-side checks (no GPU) of the prefill GEMMs' persistent tile walk, through the library's own
walk function (fp8q_check_tile_walk): with A in L2 tiles walk M fastest, otherwise in bands of M
tiles; either way every 128 x 256 output tile must be visited exactly once and inside the matrix,
including ragged M, N not a multiple of 256, and a last band shorter than the others."""
import itertools

import pytest

import fp8_quantization_amax_b200 as fq

MS = [65, 128, 129, 300, 4096, 8192, 8193, 16384, 20000, 40000]
NS = [128, 256, 384, 8192, 14336, 28672, 57344]
KS = [128, 4096, 8192, 28672]


@pytest.mark.parametrize("K", KS)
def test_tile_walk_visits_every_tile_once(K):
    for M, N in itertools.product(MS, NS):
        assert fq.check_tile_walk(M, N, K) == 0, (M, N, K)


def test_tile_walk_shapes_of_the_pages_models():
    # Llama-3 8B and 70B MLP projections at prefill sizes: banded (70B, A above L2) and M-fastest (8B)
    for (M, N, K) in [(8192, 14336, 4096), (16384, 28672, 8192), (16384, 8192, 28672), (16384, 14336, 4096)]:
        assert fq.check_tile_walk(M, N, K) == 0, (M, N, K)


def test_tile_walk_rejects_non_prefill_shapes():
    assert fq.check_tile_walk(64, 128, 128) == -1
    assert fq.check_tile_walk(128, 100, 128) == -1
    assert fq.check_tile_walk(128, 128, 100) == -1
