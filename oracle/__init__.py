"""CPU oracle (test infrastructure only).

Loads fp8_oracle.c (plain C, built with gcc here) through ctypes.  Only the
test suite, the smoke check and the benchmark's CPU-baseline leg may import
this package; the GPU library never does.  The wrappers marshal numpy arrays
and split independent scale groups across threads (ctypes releases the GIL
during a foreign call); every value the method computes (codes, scales, decoded
values, products, counts) is computed in the C file.  Two wrappers are layout
permutations written here in numpy index arithmetic and nothing else:
mx_blocked_scales (the blocked MX scale layout) and pack_b_tiles (the packed
weight-tile layout), each pinned by hand-worked byte positions.

Every function cites the page passage it follows in fp8_oracle.c; the pins
that check it against the pages live in tests/test_oracle_*.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

E4M3, E5M2 = 0, 1
PER_TENSOR, GROUP_1x128, BLOCK_128x128 = 0, 1, 2
KV_PER_TENSOR, KV_PER_HEAD, KV_PER_HEAD_TOK128 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc: IEEE float, no FMA contraction, no fast-math."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i32, i64, f32, f64, u8 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_uint8
            vp = ctypes.c_void_p
            lib.orc_fmax.argtypes = [i32]
            lib.orc_fmax.restype = f32
            lib.orc_encode.argtypes = [i32, f32]
            lib.orc_encode.restype = u8
            lib.orc_encode_nearest.argtypes = [i32, f32]
            lib.orc_encode_nearest.restype = u8
            lib.orc_scale.argtypes = [i32, f32]
            lib.orc_scale.restype = f32
            lib.orc_decode_array.argtypes = [i32, vp, i64, vp]
            lib.orc_encode_array.argtypes = [i32, vp, i64, vp]
            lib.orc_encode_nearest_array.argtypes = [i32, vp, i64, vp]
            lib.orc_quantize.argtypes = [vp, i64, i64, i32, i32, vp, vp]
            lib.orc_quantize.restype = i32
            lib.orc_dequantize.argtypes = [vp, vp, i64, i64, i32, i32, vp]
            lib.orc_dequantize.restype = i32
            lib.orc_kv_quantize.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp]
            lib.orc_kv_quantize.restype = i32
            lib.orc_gemm_rows.argtypes = [vp, vp, i32, vp, vp, i32, i32, i32, i64, i64, i64, vp, i64, vp]
            lib.orc_gemm_rows.restype = i32
            lib.orc_int8_level.argtypes = [f64, f64]
            lib.orc_int8_level.restype = i32
            lib.orc_quantize_delayed.argtypes = [vp, i64, i64, i64, i32, vp, i64, i64, vp, vp, vp]
            lib.orc_quantize_delayed.restype = i32
            lib.orc_mx_exponent.argtypes = [i32, f32]
            lib.orc_mx_exponent.restype = i32
            lib.orc_quantize_mx.argtypes = [vp, i64, i64, i32, vp, vp]
            lib.orc_quantize_mx.restype = i32
            lib.orc_dequantize_mx.argtypes = [vp, vp, i64, i64, i32, vp]
            lib.orc_dequantize_mx.restype = i32
            lib.orc_gemm_mx_rows.argtypes = [vp, vp, vp, vp, i32, i32, i64, i64, i64, vp, i64, vp]
            lib.orc_gemm_mx_rows.restype = i32
            lib.orc_scale_histogram.argtypes = [vp, i64, i32, vp]
            lib.orc_scale_histogram.restype = i32
            lib.orc_count_underflow.argtypes = [vp, vp, i64, vp]
            lib.orc_count_underflow.restype = i32
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _threads(threads: int | None) -> int:
    return max(1, threads if threads else min(32, os.cpu_count() or 1))


def _parallel(n: int, fn, threads: int | None, min_chunk: int) -> None:
    nt = _threads(threads)
    if nt == 1 or n <= min_chunk:
        fn(0, n)
        return
    chunk = max(min_chunk, -(-n // (nt * 4)))
    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(lambda s: fn(s, min(chunk, n - s)), range(0, n, chunk)))


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


# ---------------------------------------------------------------- codec

def fmax(fmt: int) -> float:
    return float(_load().orc_fmax(fmt))


def decode(codes: np.ndarray, fmt: int) -> np.ndarray:
    """uint8 codes -> exact float32 values (NaN codes keep their mantissa as payload)."""
    c = np.ascontiguousarray(codes, np.uint8)
    out = np.empty(c.shape, np.float32)
    _load().orc_decode_array(fmt, _p(c), c.size, _p(out))
    return out


def encode(q: np.ndarray, fmt: int, threads: int | None = None) -> np.ndarray:
    """float32 -> codes, bit-level round-to-nearest-even with saturation."""
    q = np.ascontiguousarray(q, np.float32)
    out = np.empty(q.shape, np.uint8)
    qf, of = q.reshape(-1), out.reshape(-1)
    lib = _load()
    _parallel(qf.size, lambda s, c: lib.orc_encode_array(fmt, _p(qf[s:s + c]), c, _p(of[s:s + c])),
              threads, 1 << 22)
    return out


def encode_nearest(q: np.ndarray, fmt: int, threads: int | None = None) -> np.ndarray:
    """float32 -> codes by brute-force nearest-value search (independent encoder)."""
    q = np.ascontiguousarray(q, np.float32)
    out = np.empty(q.shape, np.uint8)
    qf, of = q.reshape(-1), out.reshape(-1)
    lib = _load()
    _parallel(qf.size, lambda s, c: lib.orc_encode_nearest_array(fmt, _p(qf[s:s + c]), c, _p(of[s:s + c])),
              threads, 1 << 18)
    return out


def scale(amax: float, fmt: int) -> float:
    return float(_load().orc_scale(fmt, amax))


def int8_level(x: float, amax: float) -> int:
    return int(_load().orc_int8_level(x, amax))


# ---------------------------------------------------------------- quantize / dequantize

def num_scales(rows: int, cols: int, gran: int) -> int:
    if gran == PER_TENSOR:
        return 1
    if gran == GROUP_1x128:
        return cdiv(cols, 128) * rows
    return cdiv(rows, 128) * cdiv(cols, 128)


def scale_shape(rows: int, cols: int, gran: int):
    if gran == PER_TENSOR:
        return (1,)
    if gran == GROUP_1x128:
        return (cdiv(cols, 128), rows)
    return (cdiv(rows, 128), cdiv(cols, 128))


def quantize(x_bf16: np.ndarray, fmt: int, gran: int, threads: int | None = None):
    """bf16 bits [rows][cols] -> (codes uint8 [rows][cols], scales float32 in the library layout)."""
    x = np.ascontiguousarray(x_bf16, np.uint16)
    rows, cols = x.shape
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty(scale_shape(rows, cols, gran), np.float32)
    lib = _load()
    if gran == PER_TENSOR:
        rc = lib.orc_quantize(_p(x), rows, cols, fmt, gran, _p(codes), _p(scales))
        assert rc == 0
    elif gran == GROUP_1x128:
        def run(r0, n):
            s = np.empty((cdiv(cols, 128), n), np.float32)
            assert lib.orc_quantize(_p(x[r0:r0 + n]), n, cols, fmt, gran, _p(codes[r0:r0 + n]), _p(s)) == 0
            scales[:, r0:r0 + n] = s
        _parallel(rows, run, threads, 64)
    elif gran == BLOCK_128x128:
        nbr = cdiv(rows, 128)

        def run(b0, nb):
            r0, r1 = b0 * 128, min(rows, (b0 + nb) * 128)
            assert lib.orc_quantize(_p(x[r0:r1]), r1 - r0, cols, fmt, gran, _p(codes[r0:r1]),
                                    _p(scales[b0:b0 + nb])) == 0
        _parallel(nbr, run, threads, 1)
    else:
        raise ValueError(gran)
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, fmt: int, gran: int) -> np.ndarray:
    """codes [rows][cols] + scales -> bf16 bits [rows][cols]."""
    c = np.ascontiguousarray(codes, np.uint8)
    s = np.ascontiguousarray(scales, np.float32)
    rows, cols = c.shape
    y = np.empty((rows, cols), np.uint16)
    assert _load().orc_dequantize(_p(c), _p(s), rows, cols, fmt, gran, _p(y)) == 0
    return y


def kv_scale_shape(tokens: int, heads: int, gran: int):
    if gran == KV_PER_TENSOR:
        return (1,)
    if gran == KV_PER_HEAD:
        return (heads,)
    return (cdiv(tokens, 128), heads)


def kv_quantize(k_bf16: np.ndarray, v_bf16: np.ndarray, fmt: int, gran: int):
    """K, V [tokens][heads][head_dim] bf16 bits -> (k_codes, v_codes, k_scales, v_scales)."""
    k = np.ascontiguousarray(k_bf16, np.uint16)
    v = np.ascontiguousarray(v_bf16, np.uint16)
    T, H, D = k.shape
    kc, vc = np.empty(k.shape, np.uint8), np.empty(v.shape, np.uint8)
    ks = np.empty(kv_scale_shape(T, H, gran), np.float32)
    vs = np.empty(kv_scale_shape(T, H, gran), np.float32)
    rc = _load().orc_kv_quantize(_p(k), _p(v), T, H, D, fmt, gran, _p(kc), _p(vc), _p(ks), _p(vs))
    assert rc == 0
    return kc, vc, ks, vs


# ---------------------------------------------------------------- delayed scaling

def quantize_delayed(x_bf16: np.ndarray, fmt: int, history: np.ndarray, step: int, counts: np.ndarray | None = None):
    """Delayed-scaling quantization of bf16 bits x [rows][ngroups * gw] with one scale group per
    column block of gw columns, ngroups = history.shape[1].

    history float32 [H][ngroups] is read (step >= 1) and then updated in place: slot step % H
    receives this call's amax.  counts (uint64 [2], optional) accumulates saturated and
    underflowed elements.  Returns (codes uint8 like x, scales float32 [ngroups]).
    """
    x = np.ascontiguousarray(x_bf16, np.uint16)
    rows = x.shape[0]
    cols = int(np.prod(x.shape[1:])) if x.ndim > 1 else x.shape[0]
    if x.ndim == 1:
        rows = 1
    assert history.dtype == np.float32 and history.flags["C_CONTIGUOUS"] and history.ndim == 2
    H, ngroups = history.shape
    assert cols % ngroups == 0
    codes = np.empty(x.shape, np.uint8)
    scales = np.empty((ngroups,), np.float32)
    cnt = counts if counts is not None else None
    if cnt is not None:
        assert cnt.dtype == np.uint64 and cnt.shape == (2,)
    rc = _load().orc_quantize_delayed(_p(x), rows, ngroups, cols // ngroups, fmt, _p(history), H, step,
                                      _p(codes), _p(scales), _p(cnt) if cnt is not None else None)
    assert rc == 0
    return codes, scales


# ---------------------------------------------------------------- MXFP8 (1x32, power-of-two scales)

def mx_exponent(amax: float, fmt: int) -> int:
    """Smallest k with amax <= FMAX * 2^k (clamped at -127; 128 for NaN / Inf amax)."""
    return int(_load().orc_mx_exponent(fmt, float(amax)))


def quantize_mx(x_bf16: np.ndarray, fmt: int, threads: int | None = None):
    """bf16 bits [rows][cols] (cols % 32 == 0) -> (codes uint8 [rows][cols], scales uint8 [rows][cols/32])."""
    x = np.ascontiguousarray(x_bf16, np.uint16)
    rows, cols = x.shape
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, cols // 32), np.uint8)
    lib = _load()

    def run(r0, n):
        assert lib.orc_quantize_mx(_p(x[r0:r0 + n]), n, cols, fmt, _p(codes[r0:r0 + n]), _p(scales[r0:r0 + n])) == 0
    _parallel(rows, run, threads, 64)
    return codes, scales


def dequantize_mx(codes: np.ndarray, scales: np.ndarray, fmt: int) -> np.ndarray:
    c = np.ascontiguousarray(codes, np.uint8)
    s = np.ascontiguousarray(scales, np.uint8)
    rows, cols = c.shape
    y = np.empty((rows, cols), np.uint16)
    assert _load().orc_dequantize_mx(_p(c), _p(s), rows, cols, fmt, _p(y)) == 0
    return y


def mx_blocked_bytes(rows: int, cols: int) -> int:
    """Size of the blocked MX scale layout: one 512-byte chunk per 128 rows x 128 columns."""
    return cdiv(rows, 128) * cdiv(cols, 128) * 512


def mx_blocked_scales(scales: np.ndarray) -> np.ndarray:
    """Row-major MX scale bytes [rows][cols/32] -> the blocked layout the tensor cores' block-scaled
    MMA reads (one 512-byte chunk per 128 rows x 4 scale columns, chunks ordered row block by row
    block with the K blocks inside; in a chunk, byte 16*(r % 32) + 4*((r % 128) // 32) + (j % 4)
    holds scale (r, j)).  Padding rows and columns hold byte 0."""
    s = np.ascontiguousarray(scales, np.uint8)
    rows, ng = s.shape
    nrb, nkb = cdiv(rows, 128), cdiv(ng, 4)
    out = np.zeros(nrb * nkb * 512, np.uint8)
    r, j = np.indices((rows, ng))
    off = ((r // 128) * nkb + j // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + (j % 4)
    out[off] = s
    return out


def gemm_mx_rows(a_codes, sa, b_codes, sb, rows, fmt_a: int = E4M3, fmt_b: int = E4M3,
                 threads: int | None = None) -> np.ndarray:
    """fp64 rows of the MXFP8 product C = (A * 2^(sA-127)) @ (B * 2^(sB-127))^T, scales row-major
    [rows][K/32] bytes, for the listed row indices -> [len(rows)][N]."""
    A = np.ascontiguousarray(a_codes, np.uint8)
    B = np.ascontiguousarray(b_codes, np.uint8)
    sA = np.ascontiguousarray(sa, np.uint8)
    sB = np.ascontiguousarray(sb, np.uint8)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2 and K % 32 == 0 and sA.shape == (M, K // 32) and sB.shape == (N, K // 32)
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.empty((rows.size, N), np.float64)
    lib = _load()

    def run(i0, n):
        assert lib.orc_gemm_mx_rows(_p(A), _p(sA), _p(B), _p(sB), fmt_a, fmt_b, M, N, K,
                                    _p(rows[i0:i0 + n]), n, _p(out[i0:i0 + n])) == 0
    _parallel(rows.size, run, threads, 4)
    return out


def scale_histogram(scales: np.ndarray) -> np.ndarray:
    """256-bucket histogram of scales by power of two: fp32 scales by their biased exponent
    field, MX scale bytes (uint8) by value."""
    s = np.ascontiguousarray(scales)
    kind = 1 if s.dtype == np.uint8 else 0
    if kind == 0:
        s = np.ascontiguousarray(s, np.float32)
    hist = np.zeros(256, np.uint32)
    assert _load().orc_scale_histogram(_p(s), s.size, kind, _p(hist)) == 0
    return hist


def count_underflow(x_bf16: np.ndarray, codes: np.ndarray) -> int:
    """Nonzero, non-NaN inputs whose code is +-0."""
    x = np.ascontiguousarray(x_bf16, np.uint16)
    c = np.ascontiguousarray(codes, np.uint8)
    assert x.size == c.size
    out = np.zeros(1, np.uint64)
    assert _load().orc_count_underflow(_p(x), _p(c), x.size, _p(out)) == 0
    return int(out[0])


def pack_b_tiles(codes: np.ndarray) -> np.ndarray:
    """B codes [N][K] (N, K multiples of 128) -> the packed tile layout: tile (nb, kb) = rows
    [128 nb, 128 nb + 128) x columns [128 kb, 128 kb + 128) is one 16384-byte block at
    16384 * (nb * K/128 + kb); inside it row r takes bytes [128 r, 128 r + 128) with its eight
    16-byte pieces in the order piece j at position j XOR (r % 8) (the 128-byte swizzle)."""
    b = np.ascontiguousarray(codes, np.uint8)
    N, K = b.shape
    assert N % 128 == 0 and K % 128 == 0
    n, k = np.indices((N, K))
    off = ((n // 128) * (K // 128) + k // 128) * 16384 + (n % 128) * 128 + (((k % 128) // 16) ^ (n % 8)) * 16 + k % 16
    out = np.empty(N * K, np.uint8)
    out[off] = b
    return out


# ---------------------------------------------------------------- GEMM

def gemm_rows(a_codes, sa, ga, b_codes, sb, gb, rows, fmt_a: int = E4M3, fmt_b: int = E4M3,
              threads: int | None = None) -> np.ndarray:
    """fp64 rows of C = dequant(A) @ dequant(B)^T for the listed row indices -> [len(rows)][N]."""
    A = np.ascontiguousarray(a_codes, np.uint8)
    B = np.ascontiguousarray(b_codes, np.uint8)
    sA = np.ascontiguousarray(sa, np.float32)
    sB = np.ascontiguousarray(sb, np.float32)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.empty((rows.size, N), np.float64)
    lib = _load()

    def run(i0, n):
        assert lib.orc_gemm_rows(_p(A), _p(sA), ga, _p(B), _p(sB), gb, fmt_a, fmt_b, M, N, K,
                                 _p(rows[i0:i0 + n]), n, _p(out[i0:i0 + n])) == 0
    _parallel(rows.size, run, threads, 4)
    return out
