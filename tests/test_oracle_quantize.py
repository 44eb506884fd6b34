"""Pins for the oracle's scaled quantize / dequantize / KV-cache quantize.

Independent checks, none of which re-types the oracle's code:
  * the worked example of the FP8 page (golden fixture): s = 10/448 sends 0.05 -> 2.25 and
    0.1 -> 4.5, while INT8 with step 10/127 sends both to level 1;
  * the page's statement that the largest element of a block maps exactly to 448;
  * brute force on tiny tensors: numpy float32 arithmetic for amax, s and x/s, and torch's
    float8 cast for the rounding, over explicitly sliced groups;
  * the rounding error bound, and locality (an element only moves its own group);
  * dequantize against torch's float8 decode, float32 product and bfloat16 rounding.
"""
import json
import os

import numpy as np
import pytest
import torch

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")
TORCH_T = {0: torch.float8_e4m3fn, 1: torch.float8_e5m2}
FMAX = {0: np.float32(448.0), 1: np.float32(57344.0)}


def f32_to_bf16_bits(v):
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_value(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).float().numpy()


def brute_group(xv: np.ndarray, fmt: int):
    """One scale group by brute force: numpy fp32 arithmetic + torch's float8 cast."""
    xv = xv.astype(np.float32)
    amax = np.max(np.abs(xv)) if xv.size else np.float32(0)
    s = np.float32(amax) / FMAX[fmt]
    if s == 0:
        return np.where(np.signbit(xv), 0x80, 0x00).astype(np.uint8), np.float32(s)
    q = np.clip(xv / s, -FMAX[fmt], FMAX[fmt]).astype(np.float32)   # saturate, then round
    codes = torch.from_numpy(q).to(TORCH_T[fmt]).view(torch.uint8).numpy()
    return codes, np.float32(s)


def brute_quantize(xb: np.ndarray, fmt: int, gran: int):
    x = bf16_value(xb)
    rows, cols = x.shape
    codes = np.zeros((rows, cols), np.uint8)
    if gran == 0:
        c, s = brute_group(x.reshape(-1), fmt)
        return c.reshape(rows, cols), np.array([s], np.float32)
    if gran == 1:
        ng = -(-cols // 128)
        scales = np.zeros((ng, rows), np.float32)
        for r in range(rows):
            for g in range(ng):
                sl = slice(g * 128, min(cols, g * 128 + 128))
                codes[r, sl], scales[g, r] = brute_group(x[r, sl], fmt)
        return codes, scales
    nbr, nbc = -(-rows // 128), -(-cols // 128)
    scales = np.zeros((nbr, nbc), np.float32)
    for i in range(nbr):
        for j in range(nbc):
            rs, cs = slice(i * 128, min(rows, i * 128 + 128)), slice(j * 128, min(cols, j * 128 + 128))
            c, scales[i, j] = brute_group(x[rs, cs].reshape(-1), fmt)
            codes[rs, cs] = c.reshape(x[rs, cs].shape)
    return codes, scales


# ------------------------------------------------------------------ worked example

def test_worked_example_fp8_vs_int8(orc):
    with open(GOLD) as f:
        g = json.load(f)
    ex = g["fp8_e4m3"]
    s = orc.scale(g["outlier"], orc.E4M3)
    assert s == np.float32(ex["scale_num"]) / np.float32(ex["scale_den"])
    for xin, want, approx in zip(ex["inputs"], ex["quantized"], ex["quotients_approx"]):
        q = np.float32(xin) / np.float32(s)
        assert abs(float(q) - approx) < 0.005
        code = orc.encode(np.array([q], np.float32), orc.E4M3)
        assert orc.decode(code, orc.E4M3)[0] == want
        assert orc.int8_level(xin, g["outlier"]) == 1 == g["int8"]["level"][0]
    # the same through the bf16 tensor path: a small tensor with the outlier, per tensor and 1x128
    vals = np.array([10.0, 0.05, 0.1, -0.05, -0.1, 0.0, 0.02, -0.07], np.float32)
    xb = f32_to_bf16_bits(vals).reshape(1, -1)
    for gran in (orc.PER_TENSOR, orc.GROUP_1x128):
        codes, scales = orc.quantize(xb, orc.E4M3, gran)
        dec = orc.decode(codes, orc.E4M3)[0]
        assert dec[0] == g["block_max_maps_to"]
        assert list(dec[1:5]) == [2.25, 4.5, -2.25, -4.5]
        assert scales.reshape(-1)[0] == np.float32(10.0) / np.float32(448.0)


# ------------------------------------------------------------------ brute force on tiny tensors

SHAPES = [(1, 8), (1, 128), (3, 136), (127, 129), (128, 128), (129, 257), (2, 1000)]


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("gran", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES)
def test_quantize_bruteforce_tiny(orc, fmt, gran, shape):
    rng = np.random.default_rng(hash((fmt, gran, shape)) & 0xFFFF)
    x = rng.standard_normal(shape).astype(np.float32) * np.float32(0.3)
    x[rng.random(shape) < 0.01] *= 40
    xb = f32_to_bf16_bits(x)
    c_or, s_or = orc.quantize(xb, fmt, gran)
    c_bf, s_bf = brute_quantize(xb, fmt, gran)
    assert s_or.shape == s_bf.shape
    assert np.array_equal(s_or.view(np.uint32), s_bf.view(np.uint32))
    assert np.array_equal(c_or, c_bf)


def test_special_groups(orc):
    """All-zero groups keep signed zeros and scale 0; subnormal bf16 inputs; ties."""
    x = np.zeros((2, 256), np.uint16)
    x[0, :128] = 0x8000                         # -0.0 everywhere in group 0 of row 0
    x[1, 128:] = 0x0001                         # the smallest bf16 subnormal, 2^-133
    x[1, 130] = 0x8003
    for fmt in (0, 1):
        c, s = orc.quantize(x, fmt, orc.GROUP_1x128)
        assert s[0, 0] == 0 and np.all(c[0, :128] == 0x80) and np.all(c[0, 128:] == 0)
        assert s[0, 1] == 0 and np.all(c[1, :128] == 0)
        cb, sb = brute_quantize(x, fmt, orc.GROUP_1x128)
        assert np.array_equal(c, cb) and np.array_equal(s.view(np.uint32), sb.view(np.uint32))


# ------------------------------------------------------------------ invariants

@pytest.mark.parametrize("fmt,maxcode", [(0, 0x7E), (1, 0x7B)])
@pytest.mark.parametrize("gran", [0, 1, 2])
def test_group_max_maps_to_format_max(orc, fmt, maxcode, gran):
    """The page: s = a/448 makes the block's largest weight land exactly on 448."""
    x = synth.weight_8b(seed=5, n=300, k=520)
    codes, scales = orc.quantize(x, fmt, gran)
    xf = np.abs(bf16_value(x))
    rows, cols = x.shape
    if gran == 0:
        groups = [(slice(0, rows), slice(0, cols))]
    elif gran == 1:
        groups = [(slice(r, r + 1), slice(g, min(cols, g + 128))) for r in range(rows) for g in range(0, cols, 128)]
    else:
        groups = [(slice(i, min(rows, i + 128)), slice(j, min(cols, j + 128)))
                  for i in range(0, rows, 128) for j in range(0, cols, 128)]
    for rs, cs in groups:
        blk = xf[rs, cs]
        r, c = np.unravel_index(np.argmax(blk), blk.shape)
        assert (codes[rs, cs][r, c] & 0x7F) == maxcode


@pytest.mark.parametrize("fmt,m", [(0, 3), (1, 2)])
def test_error_bound(orc, fmt, m):
    x = synth.activations(seed=6, m=64, k=1024)
    codes, scales = orc.quantize(x, fmt, orc.GROUP_1x128)
    xf = bf16_value(x).astype(np.float64)
    s = np.repeat(scales.T, 128, axis=1)[:, :1024].astype(np.float64)
    dec = orc.decode(codes, fmt).astype(np.float64) * s
    sub_half = 2.0 ** ((-6 if fmt == 0 else -14) - m - 1)          # half the subnormal step
    bound = np.abs(xf) * 2.0 ** (-m - 1) + s * sub_half + np.abs(xf) * 2.0 ** -23
    assert np.all(np.abs(dec - xf) <= bound)


def test_locality(orc):
    """Raising one element changes its own group's scale and codes, and nothing else."""
    x = synth.weight_8b(seed=7, n=256, k=384)
    for gran in (1, 2):
        c0, s0 = orc.quantize(x, 0, gran)
        y = x.copy()
        y[130, 200] = f32_to_bf16_bits(np.array([5.0], np.float32))[0]
        c1, s1 = orc.quantize(y, 0, gran)
        if gran == 1:
            grp = np.zeros_like(c0, bool)
            grp[130, 128:256] = True
            assert np.count_nonzero(s0 != s1) == 1 and s1[1, 130] != s0[1, 130]
        else:
            grp = np.zeros_like(c0, bool)
            grp[128:256, 128:256] = True
            assert np.count_nonzero(s0 != s1) == 1 and s1[1, 1] != s0[1, 1]
        assert np.array_equal(c0[~grp], c1[~grp])
        assert np.count_nonzero(c0[grp] != c1[grp]) > 0


# ------------------------------------------------------------------ dequantize

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("gran", [0, 1, 2])
def test_dequantize_matches_torch(orc, fmt, gran):
    x = synth.per_tensor_1024(seed=8, rows=200, cols=264)
    codes, scales = orc.quantize(x, fmt, gran)
    y = orc.dequantize(codes, scales, fmt, gran)
    rows, cols = codes.shape
    if gran == 0:
        s = np.full((rows, cols), scales[0], np.float32)
    elif gran == 1:
        s = np.repeat(scales.T, 128, axis=1)[:, :cols]
    else:
        s = np.kron(scales, np.ones((128, 128), np.float32))[:rows, :cols]
    dec = torch.from_numpy(codes).view(TORCH_T[fmt]).float()
    ref = (dec * torch.from_numpy(np.ascontiguousarray(s))).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y, ref)
    # dequantized values stay within the rounding bound of the inputs
    xf, yf = bf16_value(x).astype(np.float64), bf16_value(y).astype(np.float64)
    assert np.all(np.abs(xf - yf) <= np.abs(xf) * (2.0 ** -3 if fmt == 0 else 2.0 ** -2) + s * 2.0 ** -9)


def test_dequantize_nan_code(orc):
    codes = np.array([[0x7F, 0xFF, 0x38, 0x00] * 2], np.uint8)
    y = orc.dequantize(codes, np.array([2.0], np.float32), 0, 0)
    v = bf16_value(y)[0]
    assert np.isnan(v[0]) and np.isnan(v[1]) and v[2] == 2.0 and v[3] == 0.0


# ------------------------------------------------------------------ KV cache

def brute_kv(k, v, fmt, gran):
    out = []
    for t in (k, v):
        T, H, D = t.shape
        x = bf16_value(t)
        codes = np.zeros(t.shape, np.uint8)
        if gran == 0:
            c, s = brute_group(x.reshape(-1), fmt)
            codes, scales = c.reshape(t.shape), np.array([s], np.float32)
        elif gran == 1:
            scales = np.zeros(H, np.float32)
            for h in range(H):
                c, scales[h] = brute_group(x[:, h, :].reshape(-1), fmt)
                codes[:, h, :] = c.reshape(T, D)
        else:
            nb = -(-T // 128)
            scales = np.zeros((nb, H), np.float32)
            for b in range(nb):
                ts = slice(b * 128, min(T, b * 128 + 128))
                for h in range(H):
                    c, scales[b, h] = brute_group(x[ts, h, :].reshape(-1), fmt)
                    codes[ts, h, :] = c.reshape(x[ts, h, :].shape)
        out.append((codes, scales))
    return out


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("gran", [0, 1, 2])
@pytest.mark.parametrize("shape", [(1, 1, 8), (5, 3, 16), (130, 2, 128), (257, 8, 64)])
def test_kv_bruteforce_tiny(orc, fmt, gran, shape):
    T, H, D = shape
    k, v = synth.kv_70b(seed=9, tokens=T, heads=H, head_dim=D)
    kc, vc, ks, vs = orc.kv_quantize(k, v, fmt, gran)
    (bkc, bks), (bvc, bvs) = brute_kv(k, v, fmt, gran)
    assert np.array_equal(kc, bkc) and np.array_equal(vc, bvc)
    assert np.array_equal(ks.view(np.uint32), bks.view(np.uint32))
    assert np.array_equal(vs.view(np.uint32), bvs.view(np.uint32))


def test_kv_separate_k_and_v_scales(orc):
    """K and V get their own scales (keys are concentrated, values spread out)."""
    k, v = synth.kv_70b(seed=3, tokens=256, heads=8, head_dim=128)
    kc, vc, ks, vs = orc.kv_quantize(k, v, 0, orc.KV_PER_HEAD)
    assert not np.array_equal(ks, vs)
    # per-head key scales follow the per-head multipliers u_h ~ U(0.5, 4)
    assert ks.max() / ks.min() > 1.5
