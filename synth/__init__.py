"""Seeded synthetic input tensors (bfloat16 bit patterns as numpy uint16).

Shared by the CPU oracle's tests and by the GPU path's tests and benchmark.
It draws random numbers and lays them out as tensors; it computes nothing of
the FP8 method itself.  The generators are counter based (see synth.c), so a
tensor is produced in parallel chunks and any element can be redrawn alone.

Workload recipes follow the synthetic configurations the build is measured on
(Llama-3 8B / 70B shaped weights, activations and KV caches).  Wherever a
recipe leaves a choice open, the choice is written next to it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, IEEE float, no FMA contraction)."""
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
            i64, u64, f64 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
            vp = ctypes.c_void_p
            lib.synth_key.argtypes = [u64, u64]
            lib.synth_key.restype = u64
            lib.synth_u64.argtypes = [u64, i64, i64, vp]
            lib.synth_uniform_f64.argtypes = [u64, i64, i64, f64, f64, vp]
            lib.synth_normal_f64.argtypes = [u64, i64, i64, f64, f64, vp]
            lib.synth_uniform_bf16.argtypes = [u64, i64, i64, f64, f64, vp]
            lib.synth_normal_bf16.argtypes = [u64, i64, i64, f64, f64, vp]
            lib.synth_normal_gain_bf16.argtypes = [u64, i64, i64, i64, f64, vp, vp, vp]
            lib.synth_scale_points_normal_bf16.argtypes = [u64, f64, vp, i64, i64, i64, f64, vp]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _chunked(n: int, fn, min_chunk: int = 1 << 20) -> None:
    """Run fn(start, count) over [0, n) in parallel chunks (ctypes drops the GIL)."""
    if n <= min_chunk:
        fn(0, n)
        return
    nt = _threads()
    chunk = max(min_chunk, -(-n // (nt * 4)))
    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(lambda s: fn(s, min(chunk, n - s)), range(0, n, chunk)))


def key(seed: int, stream: int) -> int:
    return _load().synth_key(seed, stream)


def u64(k: int, n: int, start: int = 0) -> np.ndarray:
    out = np.empty(n, np.uint64)
    _load().synth_u64(k, start, n, _ptr(out))
    return out


def uniform_f64(k: int, n: int, lo: float, hi: float) -> np.ndarray:
    out = np.empty(n, np.float64)
    _load().synth_uniform_f64(k, 0, n, lo, hi, _ptr(out))
    return out


def uniform_bf16(k: int, shape, lo: float, hi: float) -> np.ndarray:
    out = np.empty(shape, np.uint16)
    flat = out.reshape(-1)
    lib = _load()
    _chunked(flat.size, lambda s, c: lib.synth_uniform_bf16(k, s, c, lo, hi, _ptr(flat[s:s + c])))
    return out


def normal_bf16(k: int, shape, std: float, row_gain: np.ndarray | None = None,
                col_gain: np.ndarray | None = None) -> np.ndarray:
    """bf16 tensor ~ N(0, std^2) * row_gain[row] * col_gain[col]; the first axis indexes rows
    and the trailing axes, flattened, index columns."""
    out = np.empty(shape, np.uint16)
    flat = out.reshape(-1)
    rows = int(shape[0]) if len(shape) else 1
    cols = flat.size // max(rows, 1)                 # all trailing axes form the columns
    rg = None if row_gain is None else np.ascontiguousarray(row_gain, np.float64)
    cg = None if col_gain is None else np.ascontiguousarray(col_gain, np.float64)
    if rg is not None and rg.size != rows:
        raise ValueError(f"row_gain has {rg.size} entries for {rows} rows")
    if cg is not None and cg.size != cols:
        raise ValueError(f"col_gain has {cg.size} entries for {cols} columns")
    lib = _load()
    if rg is None and cg is None:
        _chunked(flat.size, lambda s, c: lib.synth_normal_bf16(k, s, c, 0.0, std, _ptr(flat[s:s + c])))
    else:
        _chunked(flat.size, lambda s, c: lib.synth_normal_gain_bf16(
            k, s, c, cols, std, _ptr(rg), _ptr(cg), _ptr(flat[s:s + c])))
    return out


def distinct_indices(k: int, count: int, bound: int) -> np.ndarray:
    """`count` distinct indices in [0, bound): successive outputs mod bound, repeats skipped."""
    if count > bound:
        raise ValueError(f"cannot draw {count} distinct indices from {bound}")
    seen: dict[int, None] = {}
    i = 0
    while len(seen) < count:
        for v in u64(k, 4 * count, start=i):
            seen.setdefault(int(v % np.uint64(bound)), None)
            if len(seen) == count:
                break
        i += 4 * count
    return np.fromiter(seen.keys(), np.int64, count)


def scale_points(out: np.ndarray, k: int, std: float, idx: np.ndarray, gain: float) -> None:
    """Overwrite flat elements idx of an N(0, std^2) tensor drawn from stream k with gain x their draw."""
    flat = out.reshape(-1)
    idx = np.ascontiguousarray(idx, np.int64)
    _load().synth_scale_points_normal_bf16(k, std, _ptr(idx), idx.size, 0, flat.size, gain, _ptr(flat))


# --------------------------------------------------------------------------------------------
# Workload recipes.  Seeds: the configuration index (0..4).  Each tensor draws from its own
# stream so that a recipe can be regenerated piece by piece.


def per_tensor_1024(seed: int = 0, rows: int = 1024, cols: int = 1024) -> np.ndarray:
    """1024x1024 bf16: every entry ~ U(-0.1, 0.1), then 64 distinct positions overwritten
    with outliers of magnitude ~ U(5, 10) and a random sign (smaller shapes: one outlier per
    16 elements at most)."""
    x = uniform_bf16(key(seed, 0), (rows, cols), -0.1, 0.1)
    n_out = min(64, rows * cols // 16)
    if n_out == 0:
        return x
    pos = distinct_indices(key(seed, 1), n_out, rows * cols)
    mag = uniform_f64(key(seed, 2), n_out, 5.0, 10.0)
    sgn = np.where(u64(key(seed, 3), n_out) & np.uint64(1), -1.0, 1.0)
    vals = (sgn * mag).astype(np.float32)
    bits = vals.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16          # float -> bf16, nearest-even
    x.reshape(-1)[pos] = bits.astype(np.uint16)
    return x


def weight_8b(seed: int = 1, n: int = 14336, k: int = 4096, std: float = 0.02,
              outlier_frac: float = 1e-4, gain: float = 20.0) -> np.ndarray:
    """Llama-3-8B up-proj shaped weight [N][K] ~ N(0, std^2); floor(N*K*1e-4) distinct
    entries multiplied by 20 (before rounding to bf16)."""
    kk = key(seed, 10)
    w = normal_bf16(kk, (n, k), std)
    n_out = int(n * k * outlier_frac)
    if n_out:
        scale_points(w, kk, std, distinct_indices(key(seed, 11), n_out, n * k), gain)
    return w


def outlier_channels(seed: int, stream: int, k: int, count: int = 8) -> np.ndarray:
    return np.sort(distinct_indices(key(seed, stream), count, k))


def activations(seed: int = 1, m: int = 8192, k: int = 4096, stream: int = 12,
                n_channels: int = 8, gain: float = 50.0) -> np.ndarray:
    """Activations [M][K] ~ N(0, 1) with `n_channels` fixed channels (columns) times 50."""
    cg = np.ones(k, np.float64)
    cg[outlier_channels(seed, stream + 1, k, n_channels)] = gain
    return normal_bf16(key(seed, stream), (m, k), 1.0, col_gain=cg)


def kv_70b(seed: int = 3, tokens: int = 131072, heads: int = 8, head_dim: int = 128):
    """Llama-3-70B GQA layer KV cache, [tokens][heads][head_dim] bf16.
    K = N(0,1) * (1.5 - t/131072) * u_h with u_h ~ U(0.5, 4) per head; V = N(0, 2^2)."""
    u_h = uniform_f64(key(seed, 21), heads, 0.5, 4.0)
    row_gain = 1.5 - np.arange(tokens, dtype=np.float64) / 131072.0
    col_gain = np.repeat(u_h, head_dim)
    k_cache = normal_bf16(key(seed, 20), (tokens, heads, head_dim), 1.0,
                          row_gain=row_gain, col_gain=col_gain)
    v_cache = normal_bf16(key(seed, 22), (tokens, heads, head_dim), 2.0)
    return k_cache, v_cache


def weight_70b(seed: int = 4, which: str = "up") -> np.ndarray:
    """Llama-3-70B MLP weight ~ N(0, 0.015^2): up/gate [28672][8192], down [8192][28672]."""
    n, k, stream = (28672, 8192, 30) if which == "up" else (8192, 28672, 31)
    return normal_bf16(key(seed, stream), (n, k), 0.015)


def activations_70b(seed: int = 4, m: int = 16384, which: str = "up") -> np.ndarray:
    """Llama-3-70B MLP input [M][K] ~ N(0,1) with 8 outlier channels x50 (K = 8192 for
    up/gate, 28672 for down)."""
    k, stream = (8192, 32) if which == "up" else (28672, 34)
    return activations(seed, m, k, stream=stream)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 values (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)
