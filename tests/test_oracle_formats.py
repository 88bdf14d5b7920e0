"""Pins of the oracle's number-format code against outside references:
torch's own float8 / bfloat16 conversions (library routines), the OCP MX
value table in tests/golden, the e2m1 -> e4m3 lossless property the V4 page
states, and exact closed forms of the scale rules."""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_e2m1():
    rows = []
    with open(os.path.join(GOLDEN, "e2m1_e4m3.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            c, v, e = line.split()
            rows.append((int(c), float(v), int(e, 16)))
    return rows


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = oracle.e4m3_value(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2  # S.1111.111 only
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e2m1_decode_matches_ocp_table_and_is_exact_in_e4m3():
    for code, value, e4 in _golden_e2m1():
        assert oracle.e2m1_value([code])[0] == value
        assert math.copysign(1, oracle.e2m1_value([code])[0]) == math.copysign(1, value)
        # lossless e2m1 -> e4m3: the E4M3 encoder maps the value to a code that decodes back exactly
        enc = int(oracle.e4m3_encode([value])[0])
        assert enc == e4
        assert oracle.e4m3_value([enc])[0] == value


def test_e8m0_decode():
    got = oracle.e8m0_value(np.arange(255, dtype=np.uint8))
    assert np.array_equal(got, [math.ldexp(1.0, c - 127) for c in range(255)])
    assert math.isnan(oracle.e8m0_value([255])[0])


def test_bf16_decode_matches_torch():
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(4096, generator=g) * 10).to(torch.bfloat16)
    codes = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_value(codes), x.float().numpy().astype(np.float64))


def test_e4m3_encode_roundtrips_every_finite_code():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        v = oracle.e4m3_value([c])[0]
        assert oracle.e4m3_encode([v])[0] == c


def test_e4m3_encode_matches_torch_rne_in_range():
    g = torch.Generator().manual_seed(2)
    v = torch.cat([torch.randn(20000, generator=g) * 50, torch.randn(5000, generator=g) * 0.01,
                   (torch.rand(5000, generator=g) * 2 - 1) * 447.0])
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(v.double().numpy())
    assert np.array_equal(got, ref)


def test_e4m3_encode_ties_to_even_and_saturates():
    vals = [oracle.e4m3_value([c])[0] for c in range(0x7F)]
    for c in range(0x7E):
        mid = 0.5 * (vals[c] + vals[c + 1])
        want = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode([mid])[0] == want
        assert oracle.e4m3_encode([-mid])[0] == 0x80 | want
    assert oracle.e4m3_encode([448.0])[0] == 0x7E
    assert oracle.e4m3_encode([464.0])[0] == 0x7E
    assert oracle.e4m3_encode([1e9])[0] == 0x7E
    assert oracle.e4m3_encode([-1e9])[0] == 0xFE
    assert oracle.e4m3_encode([1e-12])[0] == 0x00
    assert oracle.e4m3_encode([-1e-12])[0] == 0x80


def test_pow2_ceil_exp_is_minimal_power_of_two():
    rng = np.random.default_rng(3)
    for amax in np.concatenate([rng.lognormal(0, 4, 2000), [448.0, 448.0 * 8, 448.0 * 2 ** -20]]):
        e = oracle.pow2_ceil_exp(amax, 448.0)
        assert amax <= 448.0 * 2.0 ** e
        assert amax > 448.0 * 2.0 ** (e - 1)
    assert oracle.pow2_ceil_exp(448.0 * 8, 448.0) == 3
    assert oracle.pow2_ceil_exp(6.0, 6.0) == 0


def test_floor_log2_matches_frexp():
    rng = np.random.default_rng(4)
    for a in np.concatenate([rng.lognormal(0, 10, 2000), [1.0, 2.0, 0.5, 3.0 * 2 ** -60]]):
        m, e = math.frexp(a)
        assert oracle.floor_log2(a) == e - 1
        assert 2.0 ** (e - 1) <= a < 2.0 ** e


def test_act_quant_pow2_128_rules():
    rng = np.random.default_rng(5)
    v = rng.standard_normal(1024) * np.repeat(rng.lognormal(0, 3, 8), 128)
    v[128:256] = 0.0
    q, sc = oracle.quant_act("fp8_e4m3_pow2_b128", v)
    assert sc.shape == (8,)
    assert sc[1] == 127 and np.all(q[128:256] == 0)
    deq = oracle.dequant_act("fp8_e4m3_pow2_b128", q, sc)
    for b in range(8):
        blk = v[b * 128:(b + 1) * 128]
        amax = np.abs(blk).max()
        if amax == 0:
            continue
        e = int(sc[b]) - 127
        assert amax <= 448 * 2.0 ** e and amax > 448 * 2.0 ** (e - 1)
        # every element is within half an E4M3 spacing of the scaled value
        s = 2.0 ** e
        err = np.abs(deq[b * 128:(b + 1) * 128] - blk) / s
        mag = np.maximum(np.abs(blk) / s, 2.0 ** -6)
        spacing = 2.0 ** (np.floor(np.log2(mag)) - 3)
        assert np.all(err <= spacing / 2 + 1e-15)


def test_act_quant_values_on_grid_are_exact():
    # a block whose values already sit on the E4M3 grid times 2^5, with amax = 448 * 2^5
    codes = np.arange(0, 0x7F, dtype=np.uint8)[:128 // 2]
    base = oracle.e4m3_value(codes)
    v = np.concatenate([base, -base]) * 2.0 ** 5
    v[0] = 448.0 * 2 ** 5
    q, sc = oracle.quant_act("fp8_e4m3_pow2_b128", v)
    assert sc[0] == 127 + 5
    assert np.array_equal(oracle.dequant_act("fp8_e4m3_pow2_b128", q, sc), v)


def test_act_quant_mx_rules():
    rng = np.random.default_rng(6)
    v = rng.standard_normal(256) * np.repeat(rng.lognormal(0, 3, 8), 32)
    v[32:64] = 0.0
    q, sc = oracle.quant_act("mxfp8", v)
    assert sc.shape == (8,)
    assert sc[1] == 0 and np.all(q[32:64] == 0)
    for b in range(8):
        blk = v[b * 32:(b + 1) * 32]
        amax = np.abs(blk).max()
        if amax == 0:
            continue
        assert int(sc[b]) - 127 == math.frexp(amax)[1] - 1 - 8
    # saturation: amax/X lies in [256, 512), values above 448*X clamp to 448*X
    blk = np.full(32, 1.0)
    blk[0] = 1.9375 * 2 ** 8 / 256  # 1.9375 -> amax/X = 496 > 448
    q, sc = oracle.quant_act("mxfp8", blk)
    assert q[0] == 0x7E


def test_weight_value_fp8_block_scale_indexing():
    rows, cols = 256, 384
    w = np.full((2, rows, cols), 0x38, np.uint8)  # every code is 1.0
    s = np.zeros((2, rows // 128, cols // 128), np.float32)
    for e in range(2):
        for i in range(rows // 128):
            for j in range(cols // 128):
                s[e, i, j] = 2.0 ** (e * 10 + i * 3 + j)
    for e, r, c in [(0, 0, 0), (0, 127, 128), (0, 128, 127), (1, 200, 300), (1, 255, 383)]:
        got = oracle.weight_value("fp8_e4m3_b128x128", w, s, rows, cols, e, r, c)
        assert got == 2.0 ** (e * 10 + (r // 128) * 3 + c // 128)


def test_weight_value_fp4_nibble_order_and_scale():
    rows, cols = 2, 64
    w = np.zeros((1, rows, cols // 2), np.uint8)
    w[0, 1, 0] = 0x21  # col 0 -> code 1 (0.5), col 1 -> code 2 (1.0)
    w[0, 1, 16] = 0xF7  # col 32 -> code 7 (6.0), col 33 -> code 15 (-6.0)
    s = np.full((1, rows, cols // 32), 127, np.uint8)
    s[0, 1, 1] = 127 + 3
    for fmt in ("fp4_e2m1_ue8m0_b32", "mxfp4"):
        assert oracle.weight_value(fmt, w, s, rows, cols, 0, 1, 0) == 0.5
        assert oracle.weight_value(fmt, w, s, rows, cols, 0, 1, 1) == 1.0
        assert oracle.weight_value(fmt, w, s, rows, cols, 0, 1, 32) == 48.0
        assert oracle.weight_value(fmt, w, s, rows, cols, 0, 1, 33) == -48.0
        assert oracle.weight_value(fmt, w, s, rows, cols, 0, 0, 5) == 0.0
