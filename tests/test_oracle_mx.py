"""Pins for the oracle's MXFP8 quantizer (1x32 groups, power-of-two scales; CPU only).

Block scaling with blocks of 32 (api.makesence.top "LLM推理量化:FP8 versus INT8", the
Microscaling passage).  Reading: the scale of a group is the smallest power of two 2^k with
amax <= FMAX * 2^k, stored as the byte k + 127 (k >= -127); codes are FP8(RN(x / 2^k)).

Pins: the exponent at exact powers of two of FMAX and their neighbours (closed form), the clamp,
NaN / Inf; a brute force whose exponent comes from exact rational arithmetic and whose codes
come from torch's float8 cast (a library routine); the no-saturation / minimality invariants;
dequantization against torch's float8 decode.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth

FMAX = {0: 448.0, 1: 57344.0}
TORCH = {0: torch.float8_e4m3fn, 1: torch.float8_e5m2}


def exact_k(amax, fmt):
    """Smallest k with amax <= FMAX * 2^k, by rational arithmetic (clamped at -127)."""
    if np.isnan(amax) or np.isinf(amax):
        return 128
    if amax == 0:
        return -127
    a, f = Fraction(float(amax)), Fraction(FMAX[fmt])
    k = -200
    while a > f * Fraction(2) ** k:
        k += 1
    return max(k, -127)


def bf16_vals(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("fmt", [0, 1])
def test_exponent_at_powers_of_two_of_fmax(orc, fmt):
    for j in range(-20, 21):
        a = np.float32(FMAX[fmt] * 2.0 ** j)
        assert orc.mx_exponent(a, fmt) == j                                  # exactly FMAX * 2^j
        up = np.nextafter(a, np.float32(np.inf))
        assert orc.mx_exponent(up, fmt) == j + 1                             # just above it
        down = np.nextafter(a, np.float32(0))
        assert orc.mx_exponent(down, fmt) == j                               # just below it
        half = np.float32(FMAX[fmt] * 2.0 ** (j - 1))
        assert orc.mx_exponent(np.nextafter(half, np.float32(np.inf)), fmt) == j


@pytest.mark.parametrize("fmt", [0, 1])
def test_exponent_special_values(orc, fmt):
    assert orc.mx_exponent(0.0, fmt) == -127
    assert orc.mx_exponent(np.float32(1e-40), fmt) == -127                   # clamped
    assert orc.mx_exponent(float("nan"), fmt) == 128
    assert orc.mx_exponent(float("inf"), fmt) == 128
    assert orc.mx_exponent(np.float32(3.4e38), fmt) == exact_k(np.float32(3.4e38), fmt)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(1, 32), (3, 96), (17, 256)])
def test_bruteforce_tiny(orc, fmt, shape):
    rows, cols = shape
    x = synth.per_tensor_1024(seed=rows + cols, rows=rows, cols=cols)
    codes, scales = orc.quantize_mx(x, fmt)
    xf = bf16_vals(x).reshape(rows, cols // 32, 32)
    for r in range(rows):
        for g in range(cols // 32):
            grp = xf[r, g]
            k = exact_k(np.abs(grp).max(), fmt)
            assert scales[r, g] == k + 127
            q = torch.from_numpy((grp / np.float32(2.0 ** k)).astype(np.float32))
            want = q.to(TORCH[fmt]).view(torch.uint8).numpy()
            assert np.array_equal(codes[r, g * 32:(g + 1) * 32], want), (r, g)


@pytest.mark.parametrize("fmt", [0, 1])
def test_no_saturation_and_minimal_scale(orc, fmt):
    x = synth.activations(seed=3, m=64, k=512)                                # includes x50 outlier channels
    codes, scales = orc.quantize_mx(x, fmt)
    dec = orc.decode(codes, fmt).reshape(64, 16, 32)
    assert np.all(np.abs(dec) <= FMAX[fmt])
    k = scales.astype(np.int32) - 127
    amax = np.abs(bf16_vals(x)).reshape(64, 16, 32).max(axis=2)
    q = amax / np.exp2(k.astype(np.float64))
    assert np.all(q <= FMAX[fmt]) and np.all((q > FMAX[fmt] / 2) | (k == -127) | (amax == 0))


@pytest.mark.parametrize("fmt", [0, 1])
def test_dequantize_matches_torch(orc, fmt):
    rng = np.random.default_rng(fmt)
    codes = rng.integers(0, 256, (8, 64)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x12                                     # E4M3 NaN codes aside
    if fmt == 1:
        codes[(codes & 0x7C) == 0x7C] = 0x12                                 # E5M2 Inf / NaN codes aside
    scales = rng.integers(100, 150, (8, 2)).astype(np.uint8)
    y = orc.dequantize_mx(codes, scales, fmt)
    dec = torch.from_numpy(codes).view(TORCH[fmt]).float()
    s = torch.from_numpy(np.exp2(scales.astype(np.float64) - 127).astype(np.float32)).repeat_interleave(32, dim=1)
    want = (dec * s).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y, want)
