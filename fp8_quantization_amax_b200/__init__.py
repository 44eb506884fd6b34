"""FP8 (E4M3 / E5M2) scaled quantization, KV-cache quantization, dequantization and the
block-scaled FP8 GEMM on B200 (sm_100a).

A thin ctypes binding over the C ABI in include/fp8q.h (libfp8q.so, built in-tree by
``python -m fp8_quantization_amax_b200.build``).  The binding only checks and marshals
arguments: every step runs in the library's CUDA kernels on the caller's current torch
stream.  torch supplies device memory and streams; outputs that are not passed in are
allocated with torch.empty.  There is no CPU path: CPU tensors and a missing library raise.
"""
from __future__ import annotations

import ctypes
import functools
import os
import threading

import torch

__all__ = [
    "E4M3", "E5M2", "PER_TENSOR", "GROUP_1x128", "BLOCK_128x128",
    "KV_PER_TENSOR", "KV_PER_HEAD", "KV_PER_HEAD_TOK128",
    "Fp8qError", "lib", "library_path", "device_status", "num_scales", "workspace_bytes", "kv_num_scales",
    "kv_workspace_bytes", "gemm_workspace_bytes", "scale_shape", "kv_scale_shape",
    "fp8_encode", "fp8_decode", "fp8_quantize", "fp8_dequantize", "fp8_kv_quantize",
    "fp8_kv_quantize_noalloc", "fp8_gemm_blockscaled", "fp8_quantize_delayed", "fp8_kv_quantize_delayed",
    "linear_act_workspace_bytes", "fp8_linear_dynamic", "linear_fused_workspace_bytes", "fp8_linear_dynamic_fused",
    "fp8_quantize_mx", "fp8_dequantize_mx",
    "mx_blocked_scale_bytes", "fp8_quantize_mx_blocked", "fp8_gemm_mx", "fp8_pack_b_tiles",
    "fp8_gemm_blockscaled_packed", "fp8_scale_histogram", "fp8_count_underflow", "fp8_quantize_many",
    "selftest_wait_timeout", "fp8_gemm_blockscaled_to_fp8", "check_decode_split", "check_tile_walk",
]

E4M3, E5M2 = 0, 1
PER_TENSOR, GROUP_1x128, BLOCK_128x128 = 0, 1, 2
KV_PER_TENSOR, KV_PER_HEAD, KV_PER_HEAD_TOK128 = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfp8q.so")
_lock = threading.Lock()
_lib = None


class _QuantTensor(ctypes.Structure):
    """fp8q_quant_tensor of include/fp8q.h."""
    _fields_ = [("x", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("g", ctypes.c_int),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class Fp8qError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {_status_string(status)} ({status})")


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded libfp8q.so with argument types set.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise ImportError(f"{_LIB_PATH} is missing; build it with "
                                  "`python -m fp8_quantization_amax_b200.build`")
            L = ctypes.CDLL(_LIB_PATH)
            i32, i64, sz, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
            L.fp8q_status_string.argtypes = [i32]
            L.fp8q_status_string.restype = ctypes.c_char_p
            L.fp8q_version.restype = i32
            L.fp8q_device_status.restype = ctypes.c_uint32
            L.fp8q_num_scales.argtypes = [i64, i64, i32]
            L.fp8q_num_scales.restype = sz
            L.fp8q_workspace_bytes.argtypes = [i64, i64, i32]
            L.fp8q_workspace_bytes.restype = sz
            L.fp8q_kv_num_scales.argtypes = [i64, i64, i32]
            L.fp8q_kv_num_scales.restype = sz
            L.fp8q_kv_workspace_bytes.argtypes = [i64, i64, i64, i32]
            L.fp8q_kv_workspace_bytes.restype = sz
            L.fp8q_gemm_workspace_bytes.argtypes = [i64, i64, i64]
            L.fp8q_gemm_workspace_bytes.restype = sz
            L.fp8_quantize_mx.argtypes = [vp, i64, i64, i32, vp, vp, vp]
            L.fp8_dequantize_mx.argtypes = [vp, vp, i64, i64, i32, vp, vp]
            L.fp8q_mx_blocked_scale_bytes.argtypes = [i64, i64]
            L.fp8q_mx_blocked_scale_bytes.restype = sz
            L.fp8_quantize_mx_blocked.argtypes = [vp, i64, i64, i32, vp, vp, vp]
            L.fp8_gemm_mx.argtypes = [vp, vp, i32, vp, vp, i32, i64, i64, i64, vp, vp]
            L.fp8_pack_b_tiles.argtypes = [vp, i64, i64, vp, vp]
            L.fp8_scale_histogram.argtypes = [vp, i64, i32, vp, vp]
            L.fp8q_selftest_wait_timeout.argtypes = [vp]
            L.fp8q_check_decode_split.argtypes = [i64, i64, i64, i32]
            L.fp8q_check_decode_split.restype = i32
            L.fp8q_check_tile_walk.argtypes = [i64, i64, i64]
            L.fp8q_check_tile_walk.restype = i32
            L.fp8_gemm_blockscaled_to_fp8.argtypes = [vp, vp, i32, vp, vp, i32, i64, i64, i64, vp, vp, vp]
            L.fp8_gemm_blockscaled_to_fp8.restype = i32
            L.fp8q_selftest_wait_timeout.restype = i32
            L.fp8_quantize_many.argtypes = [ctypes.POINTER(_QuantTensor), i32, i32, vp]
            L.fp8_count_underflow.argtypes = [vp, vp, i64, vp, vp]
            L.fp8_gemm_blockscaled_packed.argtypes = [vp, vp, i32, vp, vp, i32, i64, i64, i64, vp, vp, sz, vp]
            L.fp8q_linear_act_workspace_bytes.argtypes = [i64, i64]
            L.fp8q_linear_act_workspace_bytes.restype = sz
            L.fp8_linear_dynamic.argtypes = [vp, i64, i64, i64, vp, vp, i32, vp, vp, sz, vp, sz, vp]
            L.fp8q_linear_fused_workspace_bytes.argtypes = [i64, i64]
            L.fp8q_linear_fused_workspace_bytes.restype = sz
            L.fp8_linear_dynamic_fused.argtypes = [vp, i64, i64, i64, vp, vp, i32, vp, vp, sz, vp]
            L.fp8_encode.argtypes = [vp, i64, i32, vp, vp]
            L.fp8_decode.argtypes = [vp, i64, i32, vp, vp]
            L.fp8_quantize.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, sz, vp]
            L.fp8_dequantize.argtypes = [vp, vp, i64, i64, i32, i32, vp, vp]
            L.fp8_kv_quantize.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, sz, vp]
            L.fp8_gemm_blockscaled.argtypes = [vp, vp, i32, vp, vp, i32, i64, i64, i64, vp, vp, sz, vp]
            L.fp8_kv_quantize_noalloc.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp]
            L.fp8_quantize_delayed.argtypes = [vp, i64, i64, i32, vp, i64, i64, vp, vp, vp, vp, sz, vp]
            L.fp8_kv_quantize_delayed.argtypes = [vp, vp, i64, i64, i64, i32, i32, vp, vp, i64, i64, vp, vp, vp, vp,
                                                  vp, vp, sz, vp]
            for fn in ("fp8_encode", "fp8_decode", "fp8_quantize", "fp8_dequantize", "fp8_kv_quantize",
                       "fp8_gemm_blockscaled", "fp8_kv_quantize_noalloc", "fp8_quantize_delayed",
                       "fp8_kv_quantize_delayed", "fp8_linear_dynamic", "fp8_linear_dynamic_fused",
                       "fp8_quantize_mx", "fp8_dequantize_mx",
                       "fp8_quantize_mx_blocked", "fp8_gemm_mx", "fp8_pack_b_tiles",
                       "fp8_gemm_blockscaled_packed", "fp8_scale_histogram", "fp8_count_underflow",
                       "fp8_quantize_many"):
                getattr(L, fn).restype = i32
            _lib = L
    return _lib


def device_status() -> int:
    """Synchronize the device; return and clear the kernels' error bits (0 = none).

    Bit 0: a bounded wait inside a kernel gave up.  Bit 1: a GEMM workspace counter was not
    zero on entry.  After any error the cached GEMM workspaces are dropped (a kernel that ended
    early may have left counters behind)."""
    status = int(lib().fp8q_device_status())
    if status:
        _gemm_ws.clear()
    return status


def _status_string(status: int) -> str:
    try:
        return lib().fp8q_status_string(status).decode()
    except Exception:  # pragma: no cover - only while reporting another error
        return "unknown"


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise Fp8qError(fn, status)


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


# ------------------------------------------------------------------ sizes

def num_scales(rows: int, cols: int, gran: int) -> int:
    return int(lib().fp8q_num_scales(rows, cols, gran))


def workspace_bytes(rows: int, cols: int, gran: int) -> int:
    return int(lib().fp8q_workspace_bytes(rows, cols, gran))


def kv_num_scales(tokens: int, heads: int, gran: int) -> int:
    return int(lib().fp8q_kv_num_scales(tokens, heads, gran))


def kv_workspace_bytes(tokens: int, heads: int, head_dim: int, gran: int) -> int:
    return int(lib().fp8q_kv_workspace_bytes(tokens, heads, head_dim, gran))


@functools.lru_cache(maxsize=256)
def gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().fp8q_gemm_workspace_bytes(M, N, K))


def scale_shape(rows: int, cols: int, gran: int) -> tuple:
    if gran == PER_TENSOR:
        return (1,)
    if gran == GROUP_1x128:
        return (_cdiv(cols, 128), rows)
    return (_cdiv(rows, 128), _cdiv(cols, 128))


def kv_scale_shape(tokens: int, heads: int, gran: int) -> tuple:
    if gran == KV_PER_TENSOR:
        return (1,)
    if gran == KV_PER_HEAD:
        return (heads,)
    return (_cdiv(tokens, 128), heads)


# ------------------------------------------------------------------ marshalling helpers

def _dev(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (this library has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_handle(device) -> int:
    """The raw cudaStream_t of the current stream on `device` (the per-call host cost matters
    for decode-sized launches, so the direct lookup is used when torch provides it)."""
    if _raw_stream is not None:
        return _raw_stream(device.index if device.index is not None else torch.cuda.current_device())
    return torch.cuda.current_stream(device).cuda_stream


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(_stream_handle(device))


def _workspace(nbytes: int, device, ws: torch.Tensor | None) -> torch.Tensor | None:
    if nbytes == 0:
        return ws
    if ws is None:
        return torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws


# A GEMM workspace's counters (its first 64 KB) must be zero before its first use and every
# successful call leaves them zero again, so one zeroed buffer per (device, stream) is kept and
# grown on demand.
_gemm_ws: dict = {}


def _gemm_workspace(nbytes: int, device, stream: int) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    key = (device.index, stream)
    buf = _gemm_ws.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _gemm_ws[key] = buf
    return buf


# ------------------------------------------------------------------ codec

def fp8_encode(q: torch.Tensor, fmt: int = E4M3, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 values -> FP8 codes (uint8), round to nearest even, saturating."""
    _dev(q, "q", torch.float32)
    out = torch.empty(q.shape, dtype=torch.uint8, device=q.device) if out is None else _dev(out, "out", torch.uint8)
    _check("fp8_encode", lib().fp8_encode(_ptr(q), q.numel(), fmt, _ptr(out), _stream(q.device)))
    return out


def fp8_decode(codes: torch.Tensor, fmt: int = E4M3, out: torch.Tensor | None = None) -> torch.Tensor:
    """FP8 codes (uint8) -> exact fp32 values."""
    _dev(codes, "codes", torch.uint8)
    out = torch.empty(codes.shape, dtype=torch.float32, device=codes.device) if out is None else \
        _dev(out, "out", torch.float32)
    _check("fp8_decode", lib().fp8_decode(_ptr(codes), codes.numel(), fmt, _ptr(out), _stream(codes.device)))
    return out


# ------------------------------------------------------------------ quantize / dequantize

def fp8_quantize(x: torch.Tensor, fmt: int = E4M3, gran: int = GROUP_1x128, codes: torch.Tensor | None = None,
                 scales: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """bf16 [rows][cols] -> (codes uint8 [rows][cols], fp32 scales in the library layout)."""
    _dev(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows][cols]")
    rows, cols = x.shape
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=x.device) if codes is None else \
        _dev(codes, "codes", torch.uint8)
    scales = torch.empty(scale_shape(rows, cols, gran), dtype=torch.float32, device=x.device) if scales is None \
        else _dev(scales, "scales", torch.float32)
    nws = workspace_bytes(rows, cols, gran)
    ws = _workspace(nws, x.device, ws)
    st = lib().fp8_quantize(_ptr(x), rows, cols, fmt, gran, _ptr(codes), _ptr(scales), _ptr(ws),
                            0 if ws is None else ws.numel() * ws.element_size(), _stream(x.device))
    _check("fp8_quantize", st)
    return codes, scales


def _counts(counts):
    if counts is None:
        return None
    if counts.dtype != torch.int64 or counts.numel() != 2 or not counts.is_cuda or not counts.is_contiguous():
        raise ValueError("counts must be a contiguous int64 CUDA tensor of 2 entries")
    return counts


def fp8_quantize_delayed(x: torch.Tensor, history: torch.Tensor, step: int, fmt: int = E4M3,
                         codes: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                         counts: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """Per-tensor delayed scaling: bf16 [rows][cols] -> (codes, scale [1]).  history fp32 [H]
    (zero-filled before step 0) is read and updated in place; counts (int64 [2], optional)
    accumulates saturated and underflowed elements."""
    _dev(x, "x", torch.bfloat16)
    _dev(history, "history", torch.float32)
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows][cols]")
    rows, cols = x.shape
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=x.device) if codes is None else \
        _dev(codes, "codes", torch.uint8)
    scale = torch.empty((1,), dtype=torch.float32, device=x.device) if scale is None else _dev(scale, "scale", torch.float32)
    counts = _counts(counts)
    ws = _workspace(workspace_bytes(rows, cols, PER_TENSOR), x.device, ws)
    st = lib().fp8_quantize_delayed(_ptr(x), rows, cols, fmt, _ptr(history), history.numel(), step, _ptr(codes),
                                    _ptr(scale), _ptr(counts), _ptr(ws), ws.numel() * ws.element_size(),
                                    _stream(x.device))
    _check("fp8_quantize_delayed", st)
    return codes, scale


def fp8_kv_quantize_delayed(k: torch.Tensor, v: torch.Tensor, k_history: torch.Tensor, v_history: torch.Tensor,
                            step: int, fmt: int = E4M3, gran: int = KV_PER_HEAD, k_codes=None, v_codes=None,
                            k_scales=None, v_scales=None, counts: torch.Tensor | None = None, ws=None):
    """KV delayed scaling (per tensor or per head): histories fp32 [H][heads] (per head) or [H]
    (per tensor), read and updated in place -> (k_codes, v_codes, k_scales, v_scales)."""
    _dev(k, "k", torch.bfloat16)
    _dev(v, "v", torch.bfloat16)
    _dev(k_history, "k_history", torch.float32)
    _dev(v_history, "v_history", torch.float32)
    if k.dim() != 3 or k.shape != v.shape:
        raise ValueError("k and v must both be [tokens][heads][head_dim]")
    T, H, D = k.shape
    per = H if gran == KV_PER_HEAD else 1
    if k_history.numel() % max(per, 1) or k_history.shape != v_history.shape:
        raise ValueError("histories must be [history_len][heads] (per head) or [history_len] (per tensor)")
    hlen = k_history.numel() // max(per, 1)
    dev = k.device
    k_codes = torch.empty(k.shape, dtype=torch.uint8, device=dev) if k_codes is None else _dev(k_codes, "k_codes", torch.uint8)
    v_codes = torch.empty(v.shape, dtype=torch.uint8, device=dev) if v_codes is None else _dev(v_codes, "v_codes", torch.uint8)
    shp = kv_scale_shape(T, H, gran)
    k_scales = torch.empty(shp, dtype=torch.float32, device=dev) if k_scales is None else _dev(k_scales, "k_scales", torch.float32)
    v_scales = torch.empty(shp, dtype=torch.float32, device=dev) if v_scales is None else _dev(v_scales, "v_scales", torch.float32)
    counts = _counts(counts)
    ws = _workspace(kv_workspace_bytes(T, H, D, gran), dev, ws)
    st = lib().fp8_kv_quantize_delayed(_ptr(k), _ptr(v), T, H, D, fmt, gran, _ptr(k_history), _ptr(v_history), hlen,
                                       step, _ptr(k_codes), _ptr(v_codes), _ptr(k_scales), _ptr(v_scales),
                                       _ptr(counts), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                       _stream(dev))
    _check("fp8_kv_quantize_delayed", st)
    return k_codes, v_codes, k_scales, v_scales


def fp8_dequantize(codes: torch.Tensor, scales: torch.Tensor, fmt: int = E4M3, gran: int = GROUP_1x128,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """codes + scales -> bf16 [rows][cols], y = bf16(decode(code) * s)."""
    _dev(codes, "codes", torch.uint8)
    _dev(scales, "scales", torch.float32)
    if codes.dim() != 2:
        raise ValueError("codes must be 2-D [rows][cols]")
    rows, cols = codes.shape
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=codes.device) if out is None else \
        _dev(out, "out", torch.bfloat16)
    st = lib().fp8_dequantize(_ptr(codes), _ptr(scales), rows, cols, fmt, gran, _ptr(out), _stream(codes.device))
    _check("fp8_dequantize", st)
    return out


def fp8_kv_quantize(k: torch.Tensor, v: torch.Tensor, fmt: int = E4M3, gran: int = KV_PER_HEAD,
                    k_codes=None, v_codes=None, k_scales=None, v_scales=None, ws=None):
    """K, V bf16 [tokens][heads][head_dim] -> (k_codes, v_codes, k_scales, v_scales)."""
    _dev(k, "k", torch.bfloat16)
    _dev(v, "v", torch.bfloat16)
    if k.dim() != 3 or k.shape != v.shape:
        raise ValueError("k and v must both be [tokens][heads][head_dim]")
    T, H, D = k.shape
    dev = k.device
    k_codes = torch.empty(k.shape, dtype=torch.uint8, device=dev) if k_codes is None else _dev(k_codes, "k_codes", torch.uint8)
    v_codes = torch.empty(v.shape, dtype=torch.uint8, device=dev) if v_codes is None else _dev(v_codes, "v_codes", torch.uint8)
    shp = kv_scale_shape(T, H, gran)
    k_scales = torch.empty(shp, dtype=torch.float32, device=dev) if k_scales is None else _dev(k_scales, "k_scales", torch.float32)
    v_scales = torch.empty(shp, dtype=torch.float32, device=dev) if v_scales is None else _dev(v_scales, "v_scales", torch.float32)
    ws = _workspace(kv_workspace_bytes(T, H, D, gran), dev, ws)
    st = lib().fp8_kv_quantize(_ptr(k), _ptr(v), T, H, D, fmt, gran, _ptr(k_codes), _ptr(v_codes), _ptr(k_scales),
                               _ptr(v_scales), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                               _stream(dev))
    _check("fp8_kv_quantize", st)
    return k_codes, v_codes, k_scales, v_scales


def fp8_kv_quantize_noalloc(k: torch.Tensor, v: torch.Tensor, fmt: int = E4M3, gran: int = KV_PER_HEAD,
                            k_codes=None, v_codes=None, k_scales=None, v_scales=None):
    """fp8_kv_quantize for callers that cannot allocate device memory: the two-pass partial maxima
    live in a fixed array inside the library (at most 32 heads for per-head scales).  Outputs
    not passed in are allocated here only for convenience; pass them to allocate nothing."""
    _dev(k, "k", torch.bfloat16)
    _dev(v, "v", torch.bfloat16)
    if k.dim() != 3 or k.shape != v.shape:
        raise ValueError("k and v must both be [tokens][heads][head_dim]")
    T, H, D = k.shape
    dev = k.device
    k_codes = torch.empty(k.shape, dtype=torch.uint8, device=dev) if k_codes is None else _dev(k_codes, "k_codes", torch.uint8)
    v_codes = torch.empty(v.shape, dtype=torch.uint8, device=dev) if v_codes is None else _dev(v_codes, "v_codes", torch.uint8)
    shp = kv_scale_shape(T, H, gran)
    k_scales = torch.empty(shp, dtype=torch.float32, device=dev) if k_scales is None else _dev(k_scales, "k_scales", torch.float32)
    v_scales = torch.empty(shp, dtype=torch.float32, device=dev) if v_scales is None else _dev(v_scales, "v_scales", torch.float32)
    st = lib().fp8_kv_quantize_noalloc(_ptr(k), _ptr(v), T, H, D, fmt, gran, _ptr(k_codes), _ptr(v_codes),
                                       _ptr(k_scales), _ptr(v_scales), _stream(dev))
    _check("fp8_kv_quantize_noalloc", st)
    return k_codes, v_codes, k_scales, v_scales


# ------------------------------------------------------------------ GEMM

def fp8_gemm_blockscaled(a: torch.Tensor, sa: torch.Tensor, b: torch.Tensor, sb: torch.Tensor,
                         ga: int = GROUP_1x128, gb: int = BLOCK_128x128, out: torch.Tensor | None = None,
                         ws: torch.Tensor | None = None) -> torch.Tensor:
    """C[M][N] (bf16) = block-scaled FP8 product of A [M][K] and B [N][K] (E4M3 codes, K-major).

    Decode shapes (M <= 64) whose weight tiles are split over several blocks need a workspace.
    Without `ws` a zero-filled buffer kept per (device, stream) is used; a caller-provided `ws`
    must have its first 64 KB (the counters) zero before its first use (every successful call
    leaves them zero) and must not be shared by calls that may overlap."""
    _dev(a, "a", torch.uint8)
    _dev(b, "b", torch.uint8)
    _dev(sa, "sa", torch.float32)
    _dev(sb, "sb", torch.float32)
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("a and b disagree on K")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device) if out is None else _dev(out, "out", torch.bfloat16)
    need = gemm_workspace_bytes(M, N, K)
    stream = _stream_handle(a.device)
    cached = ws is None
    if cached:
        ws = _gemm_workspace(need, a.device, stream)
    st = lib().fp8_gemm_blockscaled(_ptr(a), _ptr(sa), ga, _ptr(b), _ptr(sb), gb, M, N, K, _ptr(out), _ptr(ws),
                                    0 if ws is None else ws.numel() * ws.element_size(), ctypes.c_void_p(stream))
    if st != 0 and cached:
        _gemm_ws.clear()
    _check("fp8_gemm_blockscaled", st)
    return out


def fp8_gemm_blockscaled_to_fp8(a: torch.Tensor, sa: torch.Tensor, b: torch.Tensor, sb: torch.Tensor,
                                ga: int = GROUP_1x128, gb: int = BLOCK_128x128, codes: torch.Tensor | None = None,
                                scales: torch.Tensor | None = None):
    """The block-scaled GEMM (prefill shapes, M > 64) with C quantized in the epilogue:
    -> (codes uint8 [M][N], scales float32 [N/128][M]), identical to fp8_gemm_blockscaled followed
    by fp8_quantize(C, E4M3, GROUP_1x128)."""
    _dev(a, "a", torch.uint8)
    _dev(b, "b", torch.uint8)
    _dev(sa, "sa", torch.float32)
    _dev(sb, "sb", torch.float32)
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("a and b disagree on K")
    codes = torch.empty((M, N), dtype=torch.uint8, device=a.device) if codes is None else _dev(codes, "codes", torch.uint8)
    scales = torch.empty(scale_shape(M, N, GROUP_1x128), dtype=torch.float32, device=a.device) if scales is None else \
        _dev(scales, "scales", torch.float32)
    _check("fp8_gemm_blockscaled_to_fp8", lib().fp8_gemm_blockscaled_to_fp8(_ptr(a), _ptr(sa), ga, _ptr(b), _ptr(sb), gb,
                                                                           M, N, K, _ptr(codes), _ptr(scales),
                                                                           _stream(a.device)))
    return codes, scales


def fp8_pack_b_tiles(b: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """B codes [N][K] (N, K multiples of 128) -> packed tiles (uint8 [N * K]): one 16 KB block per
    128 x 128 tile in the tensor cores' swizzled shared-memory image (see fp8_gemm_blockscaled_packed)."""
    _dev(b, "b", torch.uint8)
    N, K = b.shape
    out = torch.empty(N * K, dtype=torch.uint8, device=b.device) if out is None else _dev(out, "out", torch.uint8)
    if out.numel() < N * K:
        raise ValueError(f"out needs {N * K} bytes")
    _check("fp8_pack_b_tiles", lib().fp8_pack_b_tiles(_ptr(b), N, K, _ptr(out), _stream(b.device)))
    return out


def fp8_gemm_blockscaled_packed(a: torch.Tensor, sa: torch.Tensor, bp: torch.Tensor, sb: torch.Tensor, N: int,
                                ga: int = GROUP_1x128, gb: int = BLOCK_128x128, out: torch.Tensor | None = None,
                                ws: torch.Tensor | None = None) -> torch.Tensor:
    """fp8_gemm_blockscaled with B as packed tiles (fp8_pack_b_tiles of the [N][K] codes): the same
    result; each weight tile arrives with one bulk copy.  Workspace handling as fp8_gemm_blockscaled."""
    _dev(a, "a", torch.uint8)
    _dev(bp, "bp", torch.uint8)
    _dev(sa, "sa", torch.float32)
    _dev(sb, "sb", torch.float32)
    M, K = a.shape
    if bp.numel() < N * K:
        raise ValueError("bp holds fewer than N * K bytes")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device) if out is None else _dev(out, "out", torch.bfloat16)
    need = gemm_workspace_bytes(M, N, K)
    stream = _stream_handle(a.device)
    cached = ws is None
    if cached:
        ws = _gemm_workspace(need, a.device, stream)
    st = lib().fp8_gemm_blockscaled_packed(_ptr(a), _ptr(sa), ga, _ptr(bp), _ptr(sb), gb, M, N, K, _ptr(out),
                                           _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                           ctypes.c_void_p(stream))
    if st != 0 and cached:
        _gemm_ws.clear()
    _check("fp8_gemm_blockscaled_packed", st)
    return out


def selftest_wait_timeout(device=None) -> None:
    """Launch the failure-detection self-test on the current stream: one bounded wait on a
    barrier nothing completes gives up after its time limit and sets bit 0 of device_status()."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check("fp8q_selftest_wait_timeout", lib().fp8q_selftest_wait_timeout(_stream(dev)))


def check_tile_walk(M: int, N: int, K: int) -> int:
    """Host-only check of the prefill GEMMs' tile walk: 0 when every output tile is visited exactly
    once (-1: not a prefill shape).  See fp8q_check_tile_walk in include/fp8q.h."""
    return int(lib().fp8q_check_tile_walk(M, N, K))


def check_decode_split(M: int, N: int, K: int, sms: int) -> int:
    """Host-only self-check of the decode GEMM's work split for a device with `sms` SMs (no GPU
    needed): 0 when its split-tile hand-off invariants hold, else the code of the first violation
    (-1: not a decode shape).  See fp8q_check_decode_split in include/fp8q.h."""
    return int(lib().fp8q_check_decode_split(M, N, K, sms))


def fp8_quantize_many(jobs, fmt: int = E4M3):
    """Quantize several bf16 tensors in one launch.  jobs: sequence of (x, granularity) or
    (x, granularity, codes, scales) with granularity GROUP_1x128 or BLOCK_128x128; returns a list
    of (codes, scales) identical to fp8_quantize of each."""
    if not 1 <= len(jobs) <= 8:
        raise ValueError("1 to 8 tensors per call")
    arr = (_QuantTensor * len(jobs))()
    out = []
    for j, job in enumerate(jobs):
        x, gran = job[0], job[1]
        _dev(x, "x", torch.bfloat16)
        if x.dim() != 2:
            raise ValueError("x must be 2-D [rows][cols]")
        rows, cols = x.shape
        codes = job[2] if len(job) > 2 and job[2] is not None else torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
        scales = job[3] if len(job) > 3 and job[3] is not None else torch.empty(scale_shape(rows, cols, gran),
                                                                               dtype=torch.float32, device=x.device)
        _dev(codes, "codes", torch.uint8)
        _dev(scales, "scales", torch.float32)
        arr[j] = _QuantTensor(_ptr(x), rows, cols, gran, _ptr(codes), _ptr(scales))
        out.append((codes, scales))
    _check("fp8_quantize_many", lib().fp8_quantize_many(arr, len(jobs), fmt, _stream(jobs[0][0].device)))
    return out


def fp8_scale_histogram(scales: torch.Tensor, hist: torch.Tensor | None = None) -> torch.Tensor:
    """Add a 256-bucket histogram of the scales by power of two to `hist` (int32 [256] on the
    device, created zeroed when not given): fp32 scales by their biased exponent field, MX scale
    bytes (uint8) by value."""
    if scales.dtype not in (torch.float32, torch.uint8):
        raise TypeError("scales must be float32 (fp32 scales) or uint8 (MX bytes)")
    _dev(scales, "scales", scales.dtype)
    hist = torch.zeros(256, dtype=torch.int32, device=scales.device) if hist is None else _dev(hist, "hist", torch.int32)
    kind = 0 if scales.dtype == torch.float32 else 1
    _check("fp8_scale_histogram", lib().fp8_scale_histogram(_ptr(scales), scales.numel(), kind, _ptr(hist),
                                                           _stream(scales.device)))
    return hist


def fp8_count_underflow(x: torch.Tensor, codes: torch.Tensor, count: torch.Tensor | None = None) -> torch.Tensor:
    """Add to `count` (int64 [1] on the device, created zeroed when not given) the number of
    nonzero, non-NaN bf16 inputs whose FP8 code is +-0."""
    _dev(x, "x", torch.bfloat16)
    _dev(codes, "codes", torch.uint8)
    if x.numel() != codes.numel():
        raise ValueError("x and codes differ in size")
    count = torch.zeros(1, dtype=torch.int64, device=x.device) if count is None else _dev(count, "count", torch.int64)
    _check("fp8_count_underflow", lib().fp8_count_underflow(_ptr(x), _ptr(codes), x.numel(), _ptr(count),
                                                           _stream(x.device)))
    return count


def linear_act_workspace_bytes(M: int, K: int) -> int:
    return int(lib().fp8q_linear_act_workspace_bytes(M, K))


def fp8_linear_dynamic(x: torch.Tensor, b: torch.Tensor, sb: torch.Tensor, gb: int = BLOCK_128x128,
                       out: torch.Tensor | None = None, act_ws: torch.Tensor | None = None,
                       ws: torch.Tensor | None = None) -> torch.Tensor:
    """C[M][N] (bf16) = block-scaled FP8 GEMM of the dynamically 1x128-quantized bf16 x [M][K] and
    B [N][K] (E4M3 codes): bit-identical to fp8_quantize(x, E4M3, GROUP_1x128) followed by
    fp8_gemm_blockscaled.  act_ws receives the codes and scales (allocated when not given); ws is
    the GEMM workspace (the zero-filled buffer kept per device and stream when not given)."""
    _dev(x, "x", torch.bfloat16)
    _dev(b, "b", torch.uint8)
    _dev(sb, "sb", torch.float32)
    M, K = x.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("x and b disagree on K")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else _dev(out, "out", torch.bfloat16)
    act_ws = _workspace(linear_act_workspace_bytes(M, K), x.device, act_ws)
    stream = _stream_handle(x.device)
    cached = ws is None
    if cached:
        ws = _gemm_workspace(gemm_workspace_bytes(M, N, K), x.device, stream)
    st = lib().fp8_linear_dynamic(_ptr(x), M, N, K, _ptr(b), _ptr(sb), gb, _ptr(out), _ptr(act_ws),
                                  0 if act_ws is None else act_ws.numel() * act_ws.element_size(), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(), ctypes.c_void_p(stream))
    if st != 0 and cached:
        _gemm_ws.clear()
    _check("fp8_linear_dynamic", st)
    return out


def linear_fused_workspace_bytes(M: int, K: int) -> int:
    return int(lib().fp8q_linear_fused_workspace_bytes(M, K))


def fp8_linear_dynamic_fused(x: torch.Tensor, b: torch.Tensor, sb: torch.Tensor, gb: int = BLOCK_128x128,
                             out: torch.Tensor | None = None, act_ws: torch.Tensor | None = None) -> torch.Tensor:
    """fp8_linear_dynamic at prefill shapes (M > 64) as one cooperative launch that quantizes x
    and then runs the GEMM on the codes; output bit-identical to fp8_linear_dynamic.  act_ws
    (uint8, fp8q_linear_fused_workspace_bytes(M, K) bytes) starts with two grid-barrier words
    (256 bytes) that must be zero before its first use; a buffer is allocated with them zeroed
    when not given, and every call that completes leaves them ready for the next call of any
    shape (the arrival count back at zero)."""
    _dev(x, "x", torch.bfloat16)
    _dev(b, "b", torch.uint8)
    _dev(sb, "sb", torch.float32)
    M, K = x.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("x and b disagree on K")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if out is None else _dev(out, "out", torch.bfloat16)
    nbytes = linear_fused_workspace_bytes(M, K)
    if act_ws is None and nbytes > 0:
        act_ws = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
        act_ws[:256].zero_()
    st = lib().fp8_linear_dynamic_fused(_ptr(x), M, N, K, _ptr(b), _ptr(sb), gb, _ptr(out), _ptr(act_ws),
                                        0 if act_ws is None else act_ws.numel() * act_ws.element_size(),
                                        ctypes.c_void_p(_stream_handle(x.device)))
    _check("fp8_linear_dynamic_fused", st)
    return out


def fp8_quantize_mx(x: torch.Tensor, fmt: int = E4M3, codes: torch.Tensor | None = None,
                    scales: torch.Tensor | None = None):
    """MXFP8: bf16 [rows][cols] (cols % 32 == 0) -> (codes uint8 [rows][cols], scales uint8
    [rows][cols/32] holding k + 127 for the power-of-two scale 2^k)."""
    _dev(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows][cols]")
    rows, cols = x.shape
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=x.device) if codes is None else _dev(codes, "codes", torch.uint8)
    scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device) if scales is None else \
        _dev(scales, "scales", torch.uint8)
    _check("fp8_quantize_mx", lib().fp8_quantize_mx(_ptr(x), rows, cols, fmt, _ptr(codes), _ptr(scales), _stream(x.device)))
    return codes, scales


def mx_blocked_scale_bytes(rows: int, cols: int) -> int:
    """Bytes of the blocked MX scale layout (one 512-byte chunk per 128 rows x 128 columns)."""
    return int(lib().fp8q_mx_blocked_scale_bytes(rows, cols))


def fp8_quantize_mx_blocked(x: torch.Tensor, fmt: int = E4M3, codes: torch.Tensor | None = None,
                            scales: torch.Tensor | None = None):
    """MXFP8 as fp8_quantize_mx, with the scales in the blocked layout fp8_gemm_mx reads:
    -> (codes uint8 [rows][cols], scales uint8 [mx_blocked_scale_bytes(rows, cols)])."""
    _dev(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows][cols]")
    rows, cols = x.shape
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=x.device) if codes is None else _dev(codes, "codes", torch.uint8)
    nbytes = mx_blocked_scale_bytes(rows, cols)
    scales = torch.empty(nbytes, dtype=torch.uint8, device=x.device) if scales is None else \
        _dev(scales, "scales", torch.uint8)
    if scales.numel() < nbytes:
        raise ValueError(f"scales needs {nbytes} bytes")
    _check("fp8_quantize_mx_blocked", lib().fp8_quantize_mx_blocked(_ptr(x), rows, cols, fmt, _ptr(codes), _ptr(scales),
                                                                   _stream(x.device)))
    return codes, scales


def fp8_gemm_mx(a: torch.Tensor, sa: torch.Tensor, b: torch.Tensor, sb: torch.Tensor, fa: int = E4M3,
                fb: int = E4M3, out: torch.Tensor | None = None) -> torch.Tensor:
    """C[M][N] (bf16) = MXFP8 product of A [M][K] (format fa) and B [N][K] (format fb), both with
    blocked scales (fp8_quantize_mx_blocked), on the tensor cores' block-scaled MMA."""
    _dev(a, "a", torch.uint8)
    _dev(b, "b", torch.uint8)
    _dev(sa, "sa", torch.uint8)
    _dev(sb, "sb", torch.uint8)
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("a and b disagree on K")
    if sa.numel() < mx_blocked_scale_bytes(M, K) or sb.numel() < mx_blocked_scale_bytes(N, K):
        raise ValueError("blocked scales too small")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device) if out is None else _dev(out, "out", torch.bfloat16)
    _check("fp8_gemm_mx", lib().fp8_gemm_mx(_ptr(a), _ptr(sa), fa, _ptr(b), _ptr(sb), fb, M, N, K, _ptr(out),
                                           _stream(a.device)))
    return out


def fp8_dequantize_mx(codes: torch.Tensor, scales: torch.Tensor, fmt: int = E4M3,
                      out: torch.Tensor | None = None) -> torch.Tensor:
    """MXFP8 codes + byte exponents -> bf16 [rows][cols]."""
    _dev(codes, "codes", torch.uint8)
    _dev(scales, "scales", torch.uint8)
    rows, cols = codes.shape
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=codes.device) if out is None else \
        _dev(out, "out", torch.bfloat16)
    _check("fp8_dequantize_mx", lib().fp8_dequantize_mx(_ptr(codes), _ptr(scales), rows, cols, fmt, _ptr(out),
                                                       _stream(codes.device)))
    return out
