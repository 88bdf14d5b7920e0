"""Pins of the oracle's NVFP4 path ("DeepSeek V3架构拆解…", 四 NVFP4 量化: E2M1
weights and input activations in groups of 16 with an FP8 scale each; the
shared experts stay in high precision), against things other than the oracle:
brute force over the E2M1 grid in exact arithmetic, the defining bounds of the
group scale, exhaustive E4M3 scale decoding through torch, grid fixed points,
and closed forms of one expert."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _rne_e2m1(v: float) -> int:
    a = abs(Fraction(v))
    sign = 8 if (v < 0 or (v == 0 and np.signbit(v))) else 0
    if a >= 6:
        return sign | 7
    best = min(range(8), key=lambda c: (abs(Fraction(E2M1[c]) - a), c % 2))  # ties to even code
    return sign | best


def test_e2m1_encode_matches_brute_force():
    rng = np.random.default_rng(0)
    vals = list(rng.uniform(-7, 7, 3000))
    vals += [(a + b) / 2 for a, b in zip(E2M1, E2M1[1:])]  # exact midpoints
    vals += [-(a + b) / 2 for a, b in zip(E2M1, E2M1[1:])]
    vals += [np.nextafter((a + b) / 2, 10.0) for a, b in zip(E2M1, E2M1[1:])]
    vals += [np.nextafter((a + b) / 2, -10.0) for a, b in zip(E2M1, E2M1[1:])]
    vals += E2M1 + [-x for x in E2M1] + [6.0001, 1e9, -1e9, 0.0, -0.0]
    got = oracle.e2m1_encode(vals)
    assert got.tolist() == [_rne_e2m1(v) for v in vals]


def test_e4m3_scale_codes_decode_like_torch():
    codes = np.arange(0, 0x7F, dtype=np.uint8)  # every non-negative finite E4M3 code
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(oracle.e4m3_value(codes), want)


@pytest.mark.parametrize("g", [1.0, 0.01, 3.7e-3, 2.0 ** -12])
def test_group_scale_and_codes_by_their_definition(g):
    """Each group's scale code is the E4M3 value nearest amax / (6 g) (ties to
    the even code, found by brute force over all codes), and each element the
    E2M1 value nearest v / (scale * g)."""
    rng = np.random.default_rng(int(1 / g) % 1000)
    v = rng.standard_normal(16 * 40) * np.exp2(rng.integers(-6, 6, 16 * 40)) * g * 50
    v[:16] = 0.0  # a zero group
    q, sc = oracle.quant_nvfp4(v, g)
    grid = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for b in range(40):
        blk = v[16 * b:16 * b + 16]
        t = Fraction(float(np.abs(blk).max())) / (6 * Fraction(g))
        if t >= Fraction(448):
            want_s = 0x7E
        else:
            want_s = min(range(0x7F), key=lambda c: (abs(Fraction(float(grid[c])) - t), c % 2))
        assert sc[b] == want_s, b
        s = float(grid[sc[b]])
        for i in range(16):
            want_q = 0 if s == 0 else _rne_e2m1(float(Fraction(float(blk[i])) / (Fraction(s) * Fraction(g))))
            assert q[16 * b + i] == want_q, (b, i)
    assert (q[:16] == 0).all() and sc[0] == 0
    # dequantisation: code value x scale x g
    d = oracle.dequant_nvfp4(q, sc, g)
    assert d.shape == v.shape
    mag = np.array(E2M1)[q & 7] * np.where(q & 8, -1.0, 1.0)
    assert np.array_equal(d, mag * grid[sc[np.arange(v.size) // 16]] * g)


def test_grid_values_are_fixed_points():
    """Values already on the grid (an E2M1 value times a representable scale
    times g, with the group's largest at 6) come back exactly."""
    g = 0.125
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, 64).astype(np.uint8)
    codes[::16] = 7  # each group holds a 6 so its scale is exactly s
    mag = np.array(E2M1)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    scale = 1.5  # an E4M3 value
    v = mag * scale * g
    q, sc = oracle.quant_nvfp4(v, g)
    assert np.array_equal(oracle.dequant_nvfp4(q, sc, g), v)


def test_expert_rows_one_hot_closed_form():
    """W1 = W3 = one code 1.0 at (i, h), W2 = one code 1.0 at (o, i), unit scales:
    y[o] = SiLU(x_h) x_h quantised as the intermediate, times g13^2 g2."""
    I, H = 32, 64
    one = 2  # E2M1 code of 1.0
    w13 = np.zeros((1, 2 * I, H // 2), np.uint8)
    i, h, o = 5, 9, 17
    for row in (i, I + i):
        w13[0, row, h // 2] = one if h % 2 == 0 else one << 4
    w2 = np.zeros((1, H, I // 2), np.uint8)
    w2[0, o, i // 2] = one if i % 2 == 0 else one << 4
    s13 = np.full((1, 2 * I, H // 16), 0x38, np.uint8)  # E4M3 1.0
    s2 = np.full((1, H, I // 16), 0x38, np.uint8)
    g13, g2 = np.array([0.5], np.float32), np.array([2.0], np.float32)
    xin = np.zeros((1, H))
    xin[0, h] = 3.0
    y = oracle.expert_rows_nvfp4(w13, s13, g13, w2, s2, g2, 0, I, H, xin, ga2=1.0)
    gv = 3.0 * 0.5
    a = gv / (1 + np.exp(-gv)) * gv
    q, sc = oracle.quant_nvfp4(np.r_[np.zeros(i), a, np.zeros(I - i - 1)], 1.0)
    aq = oracle.dequant_nvfp4(q, sc, 1.0)[i]
    want = np.zeros(H)
    want[o] = aq * 2.0
    assert np.allclose(y[0], want, rtol=0, atol=0)
    # linear in the down projection's tensor scale
    y2 = oracle.expert_rows_nvfp4(w13, s13, g13, w2, s2, g2 * 3, 0, I, H, xin, ga2=1.0)
    assert np.array_equal(y2, 3 * y)


def test_weight_value_decodes_nibbles_and_group_scales():
    rng = np.random.default_rng(7)
    rows, cols = 4, 64
    w = rng.integers(0, 256, (1, rows, cols // 2), dtype=np.uint8)
    s = rng.integers(0, 0x7F, (1, rows, cols // 16), dtype=np.uint8)
    g = np.array([0.75], np.float32)
    grid = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for r in range(rows):
        for c in range(cols):
            nib = (w[0, r, c // 2] >> (4 * (c % 2))) & 15
            want = E2M1[nib & 7] * (-1 if nib & 8 else 1) * grid[s[0, r, c // 16]] * 0.75
            assert oracle.weight_value_nvfp4(w, s, g, rows, cols, 0, r, c) == want
