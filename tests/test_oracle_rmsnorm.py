"""Pins of the oracle's post-attention RMSNorm (the prologue in front of the
layer: "DeepSeek V3架构拆解…", 三, decoder layer post_attention_layernorm -> MoE;
"DeepSeek-V4-Pro 架构与代码概述", 文件说明, model.py RMSNorm with an fp32
weight) and of its one-step double -> bf16 rounding, against things other than
the oracle itself: brute force over the bf16 grid in exact rational
arithmetic, a 60-digit decimal evaluation of the definition, closed forms and
exact invariances."""
import struct
from bisect import bisect_left
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _bf16_exact(code: int) -> Fraction:
    return Fraction(struct.unpack(">f", struct.pack(">I", code << 16))[0])


_POS = sorted((_bf16_exact(c), c) for c in range(0x0000, 0x7F80))  # +0 .. largest finite
_POS_VALS = [v for v, _ in _POS]
_MAX = _POS_VALS[-1]
_HALF_ULP_MAX = (_POS_VALS[-1] - _POS_VALS[-2]) / 2


def _rne_bf16(v) -> int:
    """Brute-force RNE onto the bf16 grid: nearest value, ties to the even code."""
    a = abs(Fraction(v))
    sign = 0x8000 if (Fraction(v) < 0 or (v == 0 and np.signbit(v))) else 0
    if a >= _MAX + _HALF_ULP_MAX:
        return sign | 0x7F80  # rounds past the largest finite value
    i = bisect_left(_POS_VALS, a)
    if i == len(_POS_VALS):  # above the largest finite value, below its rounding edge
        return sign | _POS[-1][1]
    if _POS_VALS[i] == a:
        return sign | _POS[i][1]
    lo, hi = _POS[i - 1], _POS[i]
    dl, dh = a - lo[0], hi[0] - a
    if dl < dh:
        c = lo[1]
    elif dh < dl:
        c = hi[1]
    else:
        c = lo[1] if lo[1] % 2 == 0 else hi[1]
    return sign | c


def test_bf16_encode_matches_brute_force():
    rng = np.random.default_rng(0)
    vals = list(rng.standard_normal(2000) * np.exp2(rng.integers(-140, 128, 2000)))
    # exact midpoints between neighbours (ties to even), and one double-ulp either side
    for c in rng.integers(1, 0x7F7F, 400):
        lo, hi = float(_bf16_exact(int(c))), float(_bf16_exact(int(c) + 1))
        mid = (lo + hi) / 2
        vals += [mid, np.nextafter(mid, 0.0), np.nextafter(mid, np.inf), -mid]
    vals += [0.0, -0.0, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -134, 2.0 ** -126, 3.3895313892515355e38,
             3.3961e38, -3.4e38, float(_MAX + _HALF_ULP_MAX), float(_MAX + _HALF_ULP_MAX) * (1 - 2 ** -50)]
    codes, _ = oracle.bf16_encode(vals)
    want = [_rne_bf16(v) for v in vals]
    assert codes.tolist() == want


def test_bf16_encode_flags_midpoints():
    lo, hi = 1.0, 1.0 + 2.0 ** -7
    mid = (lo + hi) / 2
    _, near = oracle.bf16_encode([mid, mid * (1 + 2.0 ** -40), mid * (1 + 2.0 ** -30), 1.25],
                                 tie_rel=2.0 ** -36)
    assert near.tolist() == [True, True, False, False]


def _rmsnorm_decimal(x_codes, w, eps):
    """The definition evaluated to 60 significant digits (the square root is the
    only inexact step), then rounded by brute force."""
    getcontext().prec = 60
    x = [Decimal(float(_bf16_exact(int(c)))) for c in x_codes]
    H = len(x)
    ms = sum(v * v for v in x) / Decimal(H) + Decimal(float(eps))
    r = Decimal(1) / ms.sqrt()
    return [_rne_bf16(Fraction(xv * r * Decimal(float(np.float32(wv))))) for xv, wv in zip(x, w)]


@pytest.mark.parametrize("H,eps", [(8, 1e-6), (16, 0.0), (32, 1e-2), (128, 1e-6)])
def test_rmsnorm_matches_the_definition_in_high_precision(H, eps):
    rng = np.random.default_rng(H)
    n = 6
    xf = rng.standard_normal((n, H)) * np.exp2(rng.integers(-8, 8, (n, 1)))
    x, _ = oracle.bf16_encode(xf)
    w = (1.0 + 0.2 * rng.standard_normal(H)).astype(np.float32)
    out, near = oracle.rmsnorm(x, w, eps)
    for t in range(n):
        want = _rmsnorm_decimal(x[t], w, eps)
        for h in range(H):
            if not near[t, h]:
                assert out[t, h] == want[h], (t, h)


def test_rmsnorm_closed_forms():
    H = 64
    # a constant power-of-two row with unit weight and eps = 0 normalises to +-1 exactly
    x, _ = oracle.bf16_encode(np.full((2, H), 4.0) * np.array([[1.0], [-1.0]]))
    out, _ = oracle.rmsnorm(x, np.ones(H, np.float32), 0.0)
    assert (oracle.bf16_value(out) == np.array([[1.0], [-1.0]])).all()
    # one nonzero element c in H: r = 1 / sqrt(c^2 / H + eps); y = c * r * w
    xr = np.zeros((1, H))
    xr[0, 5] = 3.0
    x, _ = oracle.bf16_encode(xr)
    w = np.full(H, 0.5, np.float32)
    out, _ = oracle.rmsnorm(x, w, 0.25)
    y = 3.0 / np.sqrt(9.0 / H + 0.25) * 0.5
    assert oracle.bf16_value(out[0, 5]) == oracle.bf16_value(oracle.bf16_encode([y])[0][0])
    assert (np.delete(oracle.bf16_value(out[0]), 5) == 0).all()
    # eps matters: with eps = 0 that element becomes 0.5 * sqrt(H)
    out0, _ = oracle.rmsnorm(x, w, 0.0)
    assert oracle.bf16_value(out0[0, 5]) == 0.5 * np.sqrt(H)


def test_rmsnorm_invariances():
    rng = np.random.default_rng(5)
    n, H = 4, 256
    x, _ = oracle.bf16_encode(rng.standard_normal((n, H)))
    w = (1 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    out, _ = oracle.rmsnorm(x, w, 0.0)
    # scaling a row by a power of two changes nothing when eps = 0 (every step is exact in scale)
    x8, _ = oracle.bf16_encode(oracle.bf16_value(x) * 2.0 ** 9)
    out8, _ = oracle.rmsnorm(x8, w, 0.0)
    assert np.array_equal(out, out8)
    # permuting the features permutes the output (the sum runs in another order, so
    # allow the near-tie elements to differ)
    p = rng.permutation(H)
    outp, nearp = oracle.rmsnorm(x[:, p], w[p], 0.0)
    ok = ~nearp
    assert np.array_equal(outp[ok], out[:, p][ok])
    # rows are independent
    out1, _ = oracle.rmsnorm(x[2:3], w, 0.0)
    assert np.array_equal(out1[0], out[2])


def test_rmsnorm_reports_a_constructed_midpoint():
    # H = 1, eps = 0: y = sign(x) * w exactly; a weight on a bf16 midpoint is a near-tie
    mid = 1.0 + 2.0 ** -8  # between 1 and 1 + 2^-7, representable in fp32
    x, _ = oracle.bf16_encode(np.array([[2.0], [-0.5]]))
    out, near = oracle.rmsnorm(x, np.array([mid], np.float32), 0.0)
    assert near.all()
    assert (oracle.bf16_value(out[:, 0]) == np.array([1.0, -1.0])).all()  # ties to even
