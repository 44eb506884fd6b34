"""Pins for the oracle's FP8 codec (encode / decode), independent of the oracle itself.

What pins it:
  * the format table and step sizes printed on the FP8 page (golden fixture);
  * torch's own float8_e4m3fn / float8_e5m2 types (a library routine) for all 256 decodes
    and, exhaustively, for every fp32 pattern in the range where the cast does not saturate;
  * a brute-force nearest-value encoder on a dense sample of patterns around every grid
    point and every midpoint, plus random patterns over the whole fp32 space;
  * the relative-error bound the page states for E4M3 (about 1/16).
"""
import json
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden", "fp8_formats.json")
TORCH_T = {0: torch.float8_e4m3fn, 1: torch.float8_e5m2}
NAME = {0: "e4m3", 1: "e5m2"}


@pytest.fixture(scope="module")
def gold():
    with open(GOLD) as f:
        return json.load(f)


def _all_codes():
    return np.arange(256, dtype=np.uint8)


def _finite_positive(orc, fmt):
    v = orc.decode(_all_codes(), fmt)
    return np.sort(v[np.isfinite(v) & (v > 0)])


@pytest.mark.parametrize("fmt", [0, 1])
def test_format_constants_match_page_table(orc, gold, fmt):
    g = gold["formats"][NAME[fmt]]
    pos = _finite_positive(orc, fmt)
    assert pos.max() == g["max"]
    assert orc.fmax(fmt) == g["max"]
    assert pos.min() == 2.0 ** g["min_subnormal_log2"]
    # smallest normal: the smallest value whose code has a nonzero exponent field
    codes = _all_codes()
    mb = g["mantissa_bits"]
    normal = orc.decode(codes[((codes >> mb) & ((1 << g["exponent_bits"]) - 1)) > 0], fmt)
    normal = normal[np.isfinite(normal) & (normal > 0)]
    assert normal.min() == 2.0 ** g["min_normal_log2"]
    # number of finite positive values: 2^(E+M) minus the reserved encodings
    n_reserved = 1 if fmt == 0 else 4
    assert pos.size == 2 ** (g["exponent_bits"] + mb) - 1 - n_reserved


def test_e4m3_has_no_infinity(orc, gold):
    v = orc.decode(_all_codes(), 0)
    assert not np.isinf(v).any()
    assert np.isnan(v).sum() == 2          # S.1111.111
    w = orc.decode(_all_codes(), 1)
    assert np.isinf(w).sum() == 2 and np.isnan(w).sum() == 6


def test_e4m3_step_sizes(orc, gold):
    pos = _finite_positive(orc, 0).astype(np.float64)
    for item in gold["e4m3_steps"]:
        lo, hi = item["interval"]
        pts = pos[(pos >= lo) & (pos <= hi)]
        assert np.all(np.diff(pts) == item["step"]), (lo, hi)
        assert pts[0] == lo and pts[-1] == hi
    s = gold["e4m3_steps_scaled"]
    for item, scaled in zip(gold["e4m3_steps"], s["steps"]):
        assert item["step"] * s["scale"] == pytest.approx(scaled)


@pytest.mark.parametrize("fmt", [0, 1])
def test_decode_matches_torch_float8(orc, fmt):
    codes = _all_codes()
    ours = orc.decode(codes, fmt)
    ref = torch.from_numpy(codes).view(TORCH_T[fmt]).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # -0 decodes with its sign
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0])


@pytest.mark.parametrize("fmt", [0, 1])
def test_roundtrip_all_256_codes(orc, fmt):
    """encode(decode(c)) == c for every code, NaN codes included.  The one exception is
    E5M2's +-Inf (0x7C / 0xFC): the cast saturates, so Inf comes back as +-57344."""
    codes = _all_codes()
    back = orc.encode(orc.decode(codes, fmt), fmt)
    if fmt == 1:
        inf = (codes & 0x7F) == 0x7C
        assert np.array_equal(back[inf], np.array([0x7B, 0xFB], np.uint8))
        codes, back = codes[~inf], back[~inf]
    assert np.array_equal(back, codes)


def _boundary_sample(orc, fmt):
    """fp32 patterns at and around (+-3 ulp) every grid value and every midpoint."""
    pos = _finite_positive(orc, fmt).astype(np.float64)
    grid = np.concatenate([[0.0], pos])
    mids = 0.5 * (grid[1:] + grid[:-1])
    # the rounding boundary above the largest value, and the top of the range
    top = np.array([pos[-1] + 0.5 * (pos[-1] - pos[-2]), pos[-1] * 2, 2.0 ** 20])
    base = np.concatenate([grid, mids, top]).astype(np.float32).view(np.int32)
    offs = np.arange(-3, 4, dtype=np.int32)
    pats = (base[:, None] + offs[None, :]).reshape(-1)
    pats = pats[pats >= 0].view(np.float32)
    return np.concatenate([pats, -pats])


def _random_patterns(n, seed):
    return np.random.default_rng(seed).integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("fmt", [0, 1])
def test_encode_equals_bruteforce_nearest(orc, fmt):
    q = np.concatenate([
        _boundary_sample(orc, fmt),
        _random_patterns(1 << 20, 1 + fmt),
        np.arange(0, 2 ** 32, 4099, dtype=np.uint64).astype(np.uint32).view(np.float32),
        np.array([np.inf, -np.inf, 0.0, -0.0, 1e30, -1e30, 3.4e38], np.float32),
    ])
    q = q[~np.isnan(q)]
    a = orc.encode(q, fmt)
    b = orc.encode_nearest(q, fmt)
    bad = np.nonzero(a != b)[0]
    assert bad.size == 0, [(float(q[i]), hex(a[i]), hex(b[i])) for i in bad[:10]]


@pytest.mark.parametrize("fmt", [0, 1])
def test_encode_matches_torch_exhaustive_in_range(orc, fmt):
    """Every positive fp32 pattern from below half the smallest subnormal up to the largest
    finite value: identical to torch's round-to-nearest-even cast (which agrees with a
    saturating cast there).  Negative values on a sample (sign symmetry)."""
    emin_sub = -9 if fmt == 0 else -16
    lo = np.float32(2.0 ** (emin_sub - 3)).view(np.uint32)
    hi = np.float32(orc.fmax(fmt)).view(np.uint32)
    chunk = 1 << 24
    tt = TORCH_T[fmt]
    for s in range(int(lo), int(hi) + 1, chunk):
        pats = np.arange(s, min(s + chunk, int(hi) + 1), dtype=np.uint32).view(np.float32)
        ours = orc.encode(pats, fmt)
        ref = torch.from_numpy(pats).to(tt).view(torch.uint8).numpy()
        bad = np.nonzero(ours != ref)[0]
        assert bad.size == 0, [(float(pats[i]), hex(ours[i]), hex(ref[i])) for i in bad[:10]]
    neg = -np.abs(_random_patterns(1 << 20, 7 + fmt))
    neg = neg[np.isfinite(neg) & (neg > -orc.fmax(fmt))]
    ref = torch.from_numpy(neg).to(tt).view(torch.uint8).numpy()
    assert np.array_equal(orc.encode(neg, fmt), ref)


@pytest.mark.parametrize("fmt,mx", [(0, 0x7E), (1, 0x7B)])
def test_saturation(orc, gold, fmt, mx):
    big = np.array([orc.fmax(fmt), orc.fmax(fmt) * 1.0001, 1e6, 3.0e38, np.inf], np.float32)
    assert np.all(orc.encode(big, fmt) == mx)
    assert np.all(orc.encode(-big, fmt) == (mx | 0x80))
    if fmt == 0:
        assert orc.decode(np.array([mx], np.uint8), 0)[0] == gold["e4m3_saturates_to"]


def test_ties_to_even_and_zero(orc):
    cases = {2.125: 2.0, 2.375: 2.5, 2.0 ** -10: 0.0, 3 * 2.0 ** -10: 2.0 ** -8, 1.0625: 1.0, 1.1875: 1.25,
             232.0: 224.0, 248.0: 256.0, 240.0: 240.0}
    q = np.array(list(cases), np.float32)
    got = orc.decode(orc.encode(q, 0), 0)
    assert np.array_equal(got, np.array(list(cases.values()), np.float32))
    z = orc.encode(np.array([-2.0 ** -10, -1e-30, -0.0], np.float32), 0)
    assert np.all(z == 0x80)


@pytest.mark.parametrize("fmt,bound", [(0, 1 / 16), (1, 1 / 8)])
def test_relative_error_bound(orc, gold, fmt, bound):
    """|dec(enc(q)) - q| <= |q| * 2^-(M+1) in the normal range; the page quotes ~1/16 for E4M3."""
    if fmt == 0:
        assert bound == gold["e4m3_relative_error_bound"]
    rng = np.random.default_rng(11)
    emin = -6 if fmt == 0 else -14
    q = (2.0 ** rng.uniform(emin, np.log2(orc.fmax(fmt)), 1 << 20)).astype(np.float32)
    err = np.abs(orc.decode(orc.encode(q, fmt), fmt).astype(np.float64) - q)
    assert np.all(err <= q.astype(np.float64) * bound)
