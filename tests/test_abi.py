"""The C-ABI library loads, exports every function include/fp8q.h declares, and rejects bad
arguments before launching anything.  No call here reaches a kernel: these run without a GPU."""
import ctypes
import os
import re

import pytest

import fp8_quantization_amax_b200 as fq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")


@pytest.fixture(scope="module")
def L():
    from fp8_quantization_amax_b200 import build
    build.build()
    return fq.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FP8Q_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ["fp8_quantize", "fp8_dequantize", "fp8_kv_quantize", "fp8_gemm_blockscaled", "fp8_encode",
               "fp8_decode", "fp8q_num_scales", "fp8q_workspace_bytes", "fp8q_status_string"]:
        assert fn in names


def test_every_declared_symbol_is_exported(L):
    for fn in declared_functions():
        assert hasattr(L, fn), fn
        assert ctypes.cast(getattr(L, fn), ctypes.c_void_p).value


def test_status_strings(L):
    for code in range(5):
        assert L.fp8q_status_string(code)
    assert L.fp8q_status_string(99) == b"unknown status"
    assert L.fp8q_version() >= 100


def test_sizes(L):
    assert fq.num_scales(8192, 4096, fq.GROUP_1x128) == 32 * 8192
    assert fq.num_scales(14336, 4096, fq.BLOCK_128x128) == 112 * 32
    assert fq.num_scales(129, 257, fq.BLOCK_128x128) == 2 * 3
    assert fq.num_scales(5, 5, fq.PER_TENSOR) == 1
    assert fq.num_scales(-1, 5, fq.PER_TENSOR) == 0
    assert fq.num_scales(5, 5, 7) == 0
    assert fq.workspace_bytes(10, 16, fq.PER_TENSOR) > 0
    assert fq.workspace_bytes(10, 16, fq.GROUP_1x128) == 0
    assert fq.kv_num_scales(131072, 8, fq.KV_PER_HEAD_TOK128) == 1024 * 8
    assert fq.kv_num_scales(131072, 8, fq.KV_PER_HEAD) == 8
    assert fq.kv_num_scales(131072, 8, fq.KV_PER_TENSOR) == 1
    assert fq.kv_workspace_bytes(131072, 8, 128, fq.KV_PER_HEAD_TOK128) == 0
    assert fq.kv_workspace_bytes(131072, 8, 128, fq.KV_PER_HEAD) >= fq.kv_workspace_bytes(131072, 8, 128, fq.KV_PER_TENSOR)
    # decode shapes (M <= 64) whose weight tiles are shared by several CTAs keep per-tile counters
    # (a fixed 64 KB region) and fp32 partial sums in the workspace (148 SMs when no GPU is
    # visible); one whole tile per CTA, larger M, or more tiles than the counters hold need none
    assert fq.gemm_workspace_bytes(16, 2048, 4096) == 65536 + 148 * 2 * 16 * 128 * 4   # two segments a CTA
    assert fq.gemm_workspace_bytes(64, 2048, 1280) == 65536 + 148 * 1 * 64 * 128 * 4
    assert fq.gemm_workspace_bytes(16, 14336, 4096) == 0       # 112 tiles: one whole tile per CTA
    assert fq.gemm_workspace_bytes(64, 128, 128) == 0          # a single unit
    assert fq.gemm_workspace_bytes(65, 14336, 4096) == 0
    assert fq.gemm_workspace_bytes(16, 128 * 20000, 128) == 0  # 20000 tiles: the prefill kernel


P = ctypes.c_void_p
# The rejection tests pass dummy device pointers that every call must refuse before launching
# anything; they run only where no GPU is visible, so a validation slip can never launch a kernel
# on those addresses.
host_only = pytest.mark.skipif(__import__("torch").cuda.is_available(),
                               reason="dummy device pointers: run on a host without a GPU")

ALIGNED = P(1 << 20)          # never dereferenced: every call below fails validation first
MISALIGNED = P((1 << 20) + 4)
ALIGNED2 = P(1 << 24)


@pytest.mark.parametrize("args,status", [
    ((ALIGNED, -1, 8, 0, 1, ALIGNED, ALIGNED, None, 0, None), 1),        # negative rows
    ((ALIGNED, 4, 12, 0, 1, ALIGNED, ALIGNED, None, 0, None), 1),        # cols % 8
    ((ALIGNED, 4, 8, 2, 1, ALIGNED, ALIGNED, None, 0, None), 1),         # bad format
    ((ALIGNED, 4, 8, 0, 3, ALIGNED, ALIGNED, None, 0, None), 1),         # bad granularity
    ((None, 4, 8, 0, 1, ALIGNED, ALIGNED, None, 0, None), 1),            # null input
    ((MISALIGNED, 4, 8, 0, 1, ALIGNED, ALIGNED, None, 0, None), 1),      # misaligned input
    ((ALIGNED, 4, 8, 0, 1, MISALIGNED, ALIGNED, None, 0, None), 1),      # misaligned codes
    ((ALIGNED, 4, 8, 0, 1, ALIGNED, None, None, 0, None), 1),            # null scales
    ((ALIGNED, 4, 8, 0, 0, ALIGNED, ALIGNED, None, 0, None), 3),         # per-tensor without workspace
    ((ALIGNED, 4, 8, 0, 0, ALIGNED, ALIGNED, ALIGNED, 16, None), 3),     # workspace too small
    ((ALIGNED, 1 << 40, 1 << 8, 0, 1, ALIGNED, ALIGNED, None, 0, None), 2),  # too large
    ((None, 0, 8, 0, 1, None, None, None, 0, None), 0),                  # empty: nothing to do
])
@host_only
def test_quantize_rejects(L, args, status):
    assert L.fp8_quantize(*args) == status


@host_only
def test_delayed_rejects(L):
    a, m = ALIGNED, MISALIGNED
    # (x, rows, cols, fmt, history, history_len, step, codes, scale, counts, ws, ws_bytes, stream)
    assert L.fp8_quantize_delayed(a, 4, 8, 0, a, 0, 1, a, a, None, a, 1 << 20, None) == 1      # empty history
    assert L.fp8_quantize_delayed(a, 4, 8, 0, a, 4, -1, a, a, None, a, 1 << 20, None) == 1     # negative step
    assert L.fp8_quantize_delayed(a, 4, 8, 0, None, 4, 1, a, a, None, a, 1 << 20, None) == 1   # null history
    assert L.fp8_quantize_delayed(a, 4, 8, 0, a, 4, 1, a, a, m, a, 1 << 20, None) == 1         # misaligned counts
    assert L.fp8_quantize_delayed(a, 4, 8, 0, a, 4, 1, a, a, None, None, 0, None) == 3         # no workspace
    assert L.fp8_quantize_delayed(a, 4, 8, 0, a, 1 << 21, 1, a, a, None, a, 1 << 20, None) == 2  # history too long
    # (k, v, T, H, D, fmt, g, kh, vh, hlen, step, kc, vc, ks, vs, counts, ws, ws_bytes, stream)
    assert L.fp8_kv_quantize_delayed(a, a, 16, 8, 128, 0, 2, a, a, 4, 1, a, a, a, a, None, a, 1 << 20, None) == 2
    assert L.fp8_kv_quantize_delayed(a, a, 16, 8, 128, 0, 1, None, a, 4, 1, a, a, a, a, None, a, 1 << 20, None) == 1
    assert L.fp8_kv_quantize_delayed(a, a, 16, 8, 128, 0, 1, a, a, 4, 1, a, a, a, a, None, None, 0, None) == 3
    assert L.fp8_kv_quantize_delayed(a, a, 16, 0, 128, 0, 1, a, a, 4, 1, a, a, a, a, None, None, 0, None) == 0


@host_only
def test_dequantize_rejects(L):
    assert L.fp8_dequantize(ALIGNED, ALIGNED, 4, 12, 0, 1, ALIGNED, None) == 1
    assert L.fp8_dequantize(ALIGNED, None, 4, 8, 0, 1, ALIGNED, None) == 1
    assert L.fp8_dequantize(ALIGNED, ALIGNED, 4, 8, 0, 1, MISALIGNED, None) == 1
    assert L.fp8_dequantize(None, None, 0, 8, 0, 1, None, None) == 0


@host_only
def test_kv_rejects(L):
    k = ALIGNED
    assert L.fp8_kv_quantize(k, k, 16, 8, 12, 0, 1, k, k, k, k, k, 1 << 20, None) == 1        # head_dim % 8
    assert L.fp8_kv_quantize(k, k, 16, 8, 128, 0, 5, k, k, k, k, k, 1 << 20, None) == 1       # bad granularity
    assert L.fp8_kv_quantize(k, k, 16, 8, 128, 0, 1, k, k, k, k, None, 0, None) == 3          # no workspace
    assert L.fp8_kv_quantize(k, k, 16, 8, 512, 0, 2, k, k, k, k, None, 0, None) == 2          # head_dim > 256
    assert L.fp8_kv_quantize(k, None, 16, 8, 128, 0, 2, k, k, k, k, None, 0, None) == 1       # null v


@host_only
def test_gemm_rejects(L):
    a = ALIGNED
    assert L.fp8_gemm_blockscaled(a, a, 1, a, a, 2, 128, 100, 128, a, None, 0, None) == 2      # N % 128
    assert L.fp8_gemm_blockscaled(a, a, 1, a, a, 2, 128, 128, 96, a, None, 0, None) == 2       # K % 128
    assert L.fp8_gemm_blockscaled(a, a, 2, a, a, 2, 128, 128, 128, a, None, 0, None) == 1      # gA
    assert L.fp8_gemm_blockscaled(a, a, 1, a, a, 1, 128, 128, 128, a, None, 0, None) == 1      # gB
    assert L.fp8_gemm_blockscaled(MISALIGNED, a, 1, a, a, 2, 128, 128, 128, a, None, 0, None) == 1
    assert L.fp8_gemm_blockscaled(a, a, 1, a, a, 2, 0, 128, 128, a, None, 0, None) == 0
    assert L.fp8_gemm_blockscaled(a, a, 1, a, a, 2, 16, 2048, 4096, a, None, 0, None) == 3      # no workspace


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        fq.fp8_quantize(torch.zeros(4, 8, dtype=torch.bfloat16))


@host_only
def test_mx_blocked_and_gemm_mx_rejects(L):
    a, m = ALIGNED, MISALIGNED
    assert L.fp8q_mx_blocked_scale_bytes(130, 256) == 2 * 2 * 512
    assert L.fp8q_mx_blocked_scale_bytes(128, 96) == 512
    assert L.fp8q_mx_blocked_scale_bytes(-1, 32) == 0
    assert L.fp8_quantize_mx_blocked(a, 4, 48, 0, a, a, None) == 1          # cols % 32
    assert L.fp8_quantize_mx_blocked(a, 4, 64, 2, a, a, None) == 1          # bad format
    assert L.fp8_quantize_mx_blocked(a, 4, 64, 0, a, None, None) == 1       # null scales
    assert L.fp8_quantize_mx_blocked(None, 0, 64, 0, None, None, None) == 0  # empty
    # (A, sA, fa, B, sB, fb, M, N, K, C, stream)
    assert L.fp8_gemm_mx(a, a, 0, a, a, 2, 16, 256, 256, a, None) == 1      # bad format
    assert L.fp8_gemm_mx(a, a, 0, a, a, 0, 16, 200, 256, a, None) == 2     # N % 128
    assert L.fp8_gemm_mx(a, a, 0, a, a, 0, 16, 256, 96, a, None) == 2      # K % 128
    assert L.fp8_gemm_mx(a, m, 0, a, a, 0, 16, 256, 256, a, None) == 1     # misaligned scales
    assert L.fp8_gemm_mx(a, a, 0, a, None, 1, 16, 256, 256, a, None) == 1  # null scales
    assert L.fp8_gemm_mx(None, None, 0, None, None, 0, 0, 256, 256, None, None) == 0


@host_only
def test_packed_b_rejects(L):
    a, m = ALIGNED, MISALIGNED
    assert L.fp8_pack_b_tiles(a, 256, 200, ALIGNED2, None) == 2       # K % 128
    assert L.fp8_pack_b_tiles(a, 100, 256, ALIGNED2, None) == 2       # N % 128
    assert L.fp8_pack_b_tiles(a, 256, 256, a, None) == 1              # in place
    assert L.fp8_pack_b_tiles(a, 256, 256, m, None) == 1              # misaligned output
    assert L.fp8_pack_b_tiles(None, 0, 256, None, None) == 0
    # (A, sA, gA, Bp, sB, gB, M, N, K, C, ws, ws_bytes, stream)
    assert L.fp8_gemm_blockscaled_packed(a, a, 2, a, a, 2, 16, 256, 256, a, a, 1 << 20, None) == 1   # gA
    assert L.fp8_gemm_blockscaled_packed(a, a, 1, a, a, 2, 16, 200, 256, a, a, 1 << 20, None) == 2   # N
    assert L.fp8_gemm_blockscaled_packed(a, a, 1, m, a, 2, 16, 256, 256, a, a, 1 << 20, None) == 1   # Bp
    assert L.fp8_gemm_blockscaled_packed(a, a, 1, a, a, 2, 16, 256, 256, a, None, 0, None) == 3      # ws


@host_only
def test_health_rejects(L):
    a, m = ALIGNED, MISALIGNED
    assert L.fp8_scale_histogram(a, 10, 2, a, None) == 1                # bad kind
    assert L.fp8_scale_histogram(P((1 << 20) + 2), 10, 0, a, None) == 1  # fp32 scales not 4-byte aligned
    assert L.fp8_scale_histogram(None, 0, 0, None, None) == 0           # empty
    assert L.fp8_count_underflow(a, m, 64, a, None) == 1                # misaligned codes
    assert L.fp8_count_underflow(a, a, -1, a, None) == 1
    assert L.fp8_count_underflow(None, None, 0, None, None) == 0


@host_only
def test_quantize_many_rejects(L):
    arr = (fq._QuantTensor * 9)()
    arr[0] = fq._QuantTensor(1 << 20, 128, 128, 0, 1 << 20, 1 << 20)
    assert L.fp8_quantize_many(arr, 1, 0, None) == 2                  # per-tensor needs two passes
    arr[0] = fq._QuantTensor(1 << 20, 128, 100, 1, 1 << 20, 1 << 20)
    assert L.fp8_quantize_many(arr, 1, 0, None) == 1                  # cols % 8
    assert L.fp8_quantize_many(arr, 9, 0, None) == 1                  # more than 8 tensors
    assert L.fp8_quantize_many(arr, 0, 0, None) == 1
    assert L.fp8_quantize_many(None, 1, 0, None) == 1
    arr[0] = fq._QuantTensor((1 << 20) + 8, 128, 128, 2, 1 << 20, 1 << 20)
    assert L.fp8_quantize_many(arr, 1, 0, None) == 1                  # x not 16-byte aligned
    arr[0] = fq._QuantTensor(None, 0, 128, 1, None, None)
    assert L.fp8_quantize_many(arr, 1, 0, None) == 0                  # empty


@host_only
def test_gemm_to_fp8_rejects(L):
    a, m = ALIGNED, MISALIGNED
    # (A, sA, gA, B, sB, gB, M, N, K, codes, scales, stream)
    assert L.fp8_gemm_blockscaled_to_fp8(a, a, 1, a, a, 2, 16, 256, 256, a, a, None) == 2     # decode shape
    assert L.fp8_gemm_blockscaled_to_fp8(a, a, 1, a, a, 2, 256, 200, 256, a, a, None) == 2    # N % 128
    assert L.fp8_gemm_blockscaled_to_fp8(a, a, 1, a, a, 2, 256, 256, 256, m, a, None) == 1    # codes alignment
    assert L.fp8_gemm_blockscaled_to_fp8(a, a, 3, a, a, 2, 256, 256, 256, a, a, None) == 1    # gA
    assert L.fp8_gemm_blockscaled_to_fp8(a, a, 1, a, a, 2, 256, 256, 256, a, None, None) == 1  # scales


@host_only
def test_linear_fused_rejects(L):
    a, m = ALIGNED, MISALIGNED
    ws = fq.linear_fused_workspace_bytes(256, 512)
    # codes (M x K, to 256) + scales (K/128 x M floats, to 256) + 256 bytes of barrier words
    assert ws == 256 * 512 + 4 * 256 * 4 + 256
    assert fq.linear_fused_workspace_bytes(64, 512) == 0          # decode shapes: not this form
    assert fq.linear_fused_workspace_bytes(300, 384) == (300 * 384 + 255) // 256 * 256 + (3 * 300 * 4 + 255) // 256 * 256 + 256
    # (X, M, N, K, B, sB, gB, C, act_ws, act_ws_bytes, stream)
    assert L.fp8_linear_dynamic_fused(a, 64, 256, 512, a, a, 2, a, a, 1 << 30, None) == 2      # decode shape
    assert L.fp8_linear_dynamic_fused(a, 256, 200, 512, a, a, 2, a, a, 1 << 30, None) == 2     # N % 128
    assert L.fp8_linear_dynamic_fused(a, 256, 256, 500, a, a, 2, a, a, 1 << 30, None) == 2     # K % 128
    assert L.fp8_linear_dynamic_fused(a, 256, 256, 512, a, a, 1, a, a, 1 << 30, None) == 1     # gB
    assert L.fp8_linear_dynamic_fused(m, 256, 256, 512, a, a, 2, a, a, 1 << 30, None) == 1     # X alignment
    assert L.fp8_linear_dynamic_fused(a, 256, 256, 512, a, a, 2, a, a, ws - 1, None) == 3      # small act_ws
    assert L.fp8_linear_dynamic_fused(a, 256, 256, 512, a, a, 2, a, P((1 << 20) + 16), ws, None) == 3  # not 256-aligned
    assert L.fp8_linear_dynamic_fused(a, 0, 256, 512, a, a, 2, a, None, 0, None) == 0          # empty
