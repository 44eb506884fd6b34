"""Pins for the oracle's delayed scaling and per-call counts (CPU only).

Delayed scaling (charles2530.github.io "量化：FP8 与混合精度推理", section "scale 是控制面";
api.makesence.top "LLM推理量化:FP8 versus INT8", section 二): the scale of step t >= 1 comes
from the amax history, s = RN(max(history) / FMAX); step 0 uses its own amax; each step
records its amax in slot t mod H.  Counts: elements that saturate, elements that underflow to
+-0 (the overflow / underflow signals of "scale 是控制面").

Pins: reductions to the dynamic quantizer (step 0, and a history holding exactly the current
amax), hand-worked values with s = 1 (a history amax equal to FMAX) where every quotient is
the input itself, the ring update, the all-zero and NaN histories, and per-head groups.
"""
import numpy as np

import synth


def _bf16(vals):
    a = np.asarray(vals, np.float32).view(np.uint32)
    keep = (a >> 16).astype(np.uint32)
    rnd = ((a & 0xFFFF) > 0x8000) | (((a & 0xFFFF) == 0x8000) & ((keep & 1) == 1))
    return (keep + rnd).astype(np.uint16)


def as_bf16_exact(vals):
    """bf16 bits of values that bf16 represents exactly (asserted)."""
    b = _bf16(vals)
    back = (b.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(back, np.asarray(vals, np.float32)), vals
    return b


def test_step0_is_the_dynamic_quantizer(orc):
    x = synth.per_tensor_1024(seed=0)
    for fmt in (orc.E4M3, orc.E5M2):
        h = np.zeros((3, 1), np.float32)
        codes, scales = orc.quantize_delayed(x, fmt, h, 0)
        ref_c, ref_s = orc.quantize(x, fmt, orc.PER_TENSOR)
        assert np.array_equal(codes, ref_c)
        assert scales.view(np.uint32)[0] == ref_s.view(np.uint32)[0]
        amax = np.abs((x.astype(np.uint32) << 16).view(np.float32)).max()
        assert h[0, 0] == amax and not h[1:].any()


def test_history_holding_the_current_amax_reduces_to_dynamic(orc):
    x = synth.normal_bf16(synth.key(5, 0), (300, 200), 2.0)
    amax = np.abs((x.astype(np.uint32) << 16).view(np.float32)).max()
    h = np.array([[0.0], [amax], [0.5 * amax]], np.float32)
    codes, scales = orc.quantize_delayed(x, orc.E4M3, h, 7)
    ref_c, ref_s = orc.quantize(x, orc.E4M3, orc.PER_TENSOR)
    assert np.array_equal(codes, ref_c) and scales[0] == ref_s[0]
    assert h[7 % 3, 0] == amax


def test_hand_worked_e4m3_unit_scale(orc):
    # history amax 448 -> s = 448 / 448 = 1 exactly, so q = x
    x = as_bf16_exact([0.5, 466.0, 464.0, -1000.0, 2.0 ** -11, 2.0 ** -10, 3 * 2.0 ** -11, 0.0, -0.0, -448.0])
    h = np.array([[448.0]], np.float32)
    cnt = np.zeros(2, np.uint64)
    codes, scales = orc.quantize_delayed(x, orc.E4M3, h, 1, counts=cnt)
    assert scales[0] == 1.0
    # 0.5 = 2^-1 -> e = 6 -> 0x30; 466 > 464 saturates; 464 is the tie between 448 (even
    # mantissa 6) and 480, so it rounds to 448 without saturating; 2^-11 < 2^-10 (half the least
    # subnormal 2^-9) -> 0; 2^-10 is the tie with 0 -> the even code 0; 3*2^-11 -> 2^-9 (0x01)
    assert codes.tolist() == [0x30, 0x7E, 0x7E, 0xFE, 0x00, 0x00, 0x01, 0x00, 0x80, 0xFE]
    assert cnt.tolist() == [2, 2]          # saturated: 466, -1000; underflowed: 2^-11, 2^-10
    assert h[0, 0] == 1000.0               # this call's amax, slot 1 % 1 = 0


def test_hand_worked_e5m2_unit_scale(orc):
    # history amax 57344 -> s = 1; E5M2 max 57344 = 1.75 * 2^15, next grid point 65536, the tie
    # 61440 goes to 65536 (57344's mantissa 11b is odd), so it saturates
    x = as_bf16_exact([61440.0, 61184.0, -65536.0, 2.0 ** -18, 2.0 ** -17, 1.5])
    h = np.array([[57344.0]], np.float32)
    cnt = np.zeros(2, np.uint64)
    codes, _ = orc.quantize_delayed(x, orc.E5M2, h, 1, counts=cnt)
    assert codes[0] == 0x7B and codes[1] == 0x7B and codes[2] == 0xFB
    assert codes[3] == 0x00 and codes[4] == 0x00          # 2^-18 < 2^-17 tie -> 0; 2^-17 tie -> even 0
    assert codes[5] == 0x3E                                # 1.5 = 1.1b * 2^0 -> e = 15, m = 2
    assert cnt.tolist() == [2, 2]


def test_ring_update_and_window_max(orc):
    H = 3
    h = np.zeros((H, 1), np.float32)
    amaxes = [4.0, 1.0, 8.0, 2.0, 0.5, 3.0]
    for t, a in enumerate(amaxes):
        x = as_bf16_exact([a, -a / 2, a / 4])
        expect_hist = a if t == 0 else max(h[:, 0])
        _, s = orc.quantize_delayed(x, orc.E4M3, h, t)
        assert s[0] == np.float32(np.float32(expect_hist) / np.float32(448.0))
        assert h[t % H, 0] == a
    assert h[:, 0].tolist() == [2.0, 0.5, 3.0]


def test_zero_history_gives_sign_only_codes(orc):
    x = as_bf16_exact([1.0, -2.0, 0.0, -0.0, 2.0 ** -100])
    h = np.zeros((2, 1), np.float32)
    cnt = np.zeros(2, np.uint64)
    codes, s = orc.quantize_delayed(x, orc.E4M3, h, 1, counts=cnt)
    assert s[0] == 0.0
    assert codes.tolist() == [0x00, 0x80, 0x00, 0x80, 0x00]
    assert cnt.tolist() == [0, 3]


def test_nan_history_is_sticky(orc):
    x = as_bf16_exact([1.0, -2.0])
    h = np.array([[1.0], [np.nan]], np.float32)
    cnt = np.zeros(2, np.uint64)
    codes, s = orc.quantize_delayed(x, orc.E4M3, h, 3, counts=cnt)
    assert np.isnan(s[0])
    assert all((c & 0x7F) == 0x7F for c in codes.tolist())
    assert cnt.tolist() == [0, 0]


def test_per_head_groups_match_the_kv_quantizer(orc):
    k, v = synth.kv_70b(seed=3, tokens=512)
    T, H, D = k.shape
    hist = np.zeros((2, H), np.float32)
    codes, scales = orc.quantize_delayed(k, orc.E4M3, hist, 0)
    kc, _, ks, _ = orc.kv_quantize(k, v, orc.E4M3, orc.KV_PER_HEAD)
    assert np.array_equal(codes, kc) and np.array_equal(scales, ks)
    amax = np.abs((k.astype(np.uint32) << 16).view(np.float32)).max(axis=(0, 2))
    assert np.array_equal(hist[0], amax) and not hist[1].any()
    # step 1 with the same tensor: history max == current amax -> the same result again
    codes1, scales1 = orc.quantize_delayed(k, orc.E4M3, hist, 1)
    assert np.array_equal(codes1, kc) and np.array_equal(scales1, ks)


def test_brute_force_tiny(orc):
    """Every element of a small tensor against a direct statement of the rule."""
    rng = np.random.default_rng(11)
    x = _bf16(rng.normal(0, 3, (4, 6)).astype(np.float32))
    h = np.array([[2.5, 0.7], [1.0, 6.0]], np.float32)
    cnt = np.zeros(2, np.uint64)
    codes, s = orc.quantize_delayed(x, orc.E4M3, h.copy(), 5, counts=cnt)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    sat = und = 0
    for g in range(2):
        sg = np.float32(np.float32(max(h[:, g])) / np.float32(448.0))
        assert s[g] == sg
        for r in range(4):
            for c in range(3):
                xv = xf[r, g * 3 + c]
                q = np.float32(xv / sg)
                assert codes[r, g * 3 + c] == orc.encode(np.array([q], np.float32), orc.E4M3)[0]
                sat += abs(float(q)) > 464.0
                und += xv != 0 and (codes[r, g * 3 + c] & 0x7F) == 0
    assert cnt.tolist() == [sat, und]
