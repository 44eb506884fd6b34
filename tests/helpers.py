"""Host <-> device marshalling for the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch


def dev_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def dev(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def nan_code_mask(codes: np.ndarray, fmt: int) -> np.ndarray:
    c = codes & 0x7F
    return c == 0x7F if fmt == 0 else (c >= 0x7D)


def assert_codes_equal(got: np.ndarray, want: np.ndarray, fmt: int, what: str = "codes"):
    """Bit-exact, except that any NaN code matches any NaN code."""
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    nan_g, nan_w = nan_code_mask(got, fmt), nan_code_mask(want, fmt)
    assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
    bad = np.nonzero((got != want) & ~nan_w)
    if bad[0].size:
        idx = tuple(b[:8] for b in bad)
        raise AssertionError(f"{what}: {bad[0].size} mismatches, first at {list(zip(*idx))}: "
                             f"got {got[idx]} want {want[idx]}")


def assert_f32_bits_equal(got: np.ndarray, want: np.ndarray, what: str = "scales"):
    """fp32 bit-exact, NaN matches NaN."""
    got = np.ascontiguousarray(got, np.float32)
    want = np.ascontiguousarray(want, np.float32)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan), f"{what}: NaN positions differ"
    bad = np.nonzero((got.view(np.uint32) != want.view(np.uint32)) & ~nan)
    if bad[0].size:
        idx = tuple(b[:8] for b in bad)
        raise AssertionError(f"{what}: {bad[0].size} mismatches, first at {list(zip(*idx))}: "
                             f"got {got[idx]} want {want[idx]}")


def assert_bf16_equal(got: np.ndarray, want: np.ndarray, what: str = "bf16"):
    got = np.asarray(got, np.uint16)
    want = np.asarray(want, np.uint16)
    nan_w = ((want & 0x7F80) == 0x7F80) & ((want & 0x7F) != 0)
    nan_g = ((got & 0x7F80) == 0x7F80) & ((got & 0x7F) != 0)
    assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
    bad = np.nonzero((got != want) & ~nan_w)
    if bad[0].size:
        idx = tuple(b[:8] for b in bad)
        raise AssertionError(f"{what}: {bad[0].size} mismatches at {list(zip(*idx))}: got {got[idx]} want {want[idx]}")
