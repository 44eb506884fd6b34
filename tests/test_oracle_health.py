"""Pins for the oracle's scale-health counts (CPU only).

charles2530.github.io "量化：FP8 与混合精度推理", "scale 是控制面": scales, overflow and underflow
should be observable.  The histogram buckets fp32 scales by power of two (biased exponent
field; zero / subnormal in bucket 0, Inf / NaN in 255) and MX scale bytes by value; the
underflow count takes nonzero, non-NaN inputs whose code is +-0.

Pins: hand-worked buckets of chosen values; the bucket of a normal scale equals the exponent
numpy's frexp gives (a library routine); hand-worked underflow cases; the count equals the
underflow count the delayed-scaling quantizer reports for the same codes.
"""
import numpy as np

import synth


def test_histogram_hand_worked(orc):
    s = np.array([1.0, 0.5, 448.0, 0.0, 1e-40, np.nan, np.inf, -2.0, 3.0], np.float32)
    h = orc.scale_histogram(s)
    want = np.zeros(256, np.uint32)
    for b in (127, 126, 135, 0, 0, 255, 255, 128, 128):
        want[b] += 1
    assert np.array_equal(h, want)
    hb = orc.scale_histogram(np.array([0, 127, 255, 127, 200], np.uint8))
    assert hb[0] == 1 and hb[127] == 2 and hb[255] == 1 and hb[200] == 1 and hb.sum() == 5


def test_histogram_matches_frexp(orc):
    rng = np.random.default_rng(5)
    s = (np.abs(rng.standard_normal(5000)) * 10.0 ** rng.uniform(-20, 20, 5000)).astype(np.float32)
    s = s[(s > np.finfo(np.float32).tiny) & np.isfinite(s)]
    _, e = np.frexp(s)                      # s = m * 2^e, m in [0.5, 1): biased exponent e - 1 + 127
    want = np.bincount(e - 1 + 127, minlength=256).astype(np.uint32)
    assert np.array_equal(orc.scale_histogram(s), want)


def test_underflow_hand_worked(orc):
    bits = lambda v: (np.float32(v).view(np.uint32) >> 16).astype(np.uint16)  # noqa: E731
    x = np.array([bits(0.0), bits(1e-10), bits(1.0), 0x7FC0, bits(-1e-10), bits(-0.0), bits(2e-10)], np.uint16)
    c = np.array([0x00, 0x80, 0x38, 0x7F, 0x01, 0x80, 0x00], np.uint8)
    assert orc.count_underflow(x, c) == 2    # 1e-10 -> -0 code and 2e-10 -> +0; zeros and NaN excluded


def test_underflow_agrees_with_delayed_counts(orc):
    x = synth.activations(seed=9, m=64, k=256)
    hist = np.zeros((2, 1), np.float32)
    hist[0, 0] = 2.0e4                       # a stale amax far above x's: many values flush to zero
    counts = np.zeros(2, np.uint64)
    codes, _ = orc.quantize_delayed(x, 0, hist, 1, counts)
    assert counts[1] > 0
    assert orc.count_underflow(x, codes) == int(counts[1])
