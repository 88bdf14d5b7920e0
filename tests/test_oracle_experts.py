"""Pins of the oracle's permutation (library stable argsort, bijection),
per-expert SwiGLU (one-hot closed forms, zero gate, linearity, block-scale
placement) and combine (identical experts reduce to a closed form)."""
import math
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def random_routing(rng, T, k, E):
    return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


# ----------------------------------------------------------------- permute
@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (64, 4, 16), (128, 8, 384), (37, 6, 7), (500, 16, 896)])
def test_permute_matches_stable_argsort(T, k, E):
    rng = np.random.default_rng(T + k + E)
    idx = random_routing(rng, T, k, min(E, max(k, E)))
    off, sp, ro = oracle.permute(idx, E)
    flat = idx.ravel()
    assert np.array_equal(sp, np.argsort(flat, kind="stable"))
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    assert np.array_equal(sp[ro], np.arange(T * k))  # round trip
    assert np.array_equal(np.sort(sp), np.arange(T * k))  # bijection
    for e in range(E):
        blk = sp[off[e]:off[e + 1]]
        assert np.all(flat[blk] == e)
        assert np.all(np.diff(blk // k) > 0)  # ascending token inside an expert


def test_permute_edge_cases():
    off, sp, ro = oracle.permute(np.zeros((0, 4), np.int32), 8)
    assert off.tolist() == [0] * 9 and sp.size == 0
    idx = np.array([[5, 1], [5, 2], [5, 0]], np.int32)  # expert 5 gets every token
    off, sp, ro = oracle.permute(idx, 6)
    assert off.tolist() == [0, 1, 2, 3, 3, 3, 6]
    assert sp.tolist() == [5, 1, 3, 0, 2, 4]
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 6]], np.int32), 6)
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, -1]], np.int32), 6)


# ----------------------------------------------------------------- experts
def silu(v):
    return v / (1.0 + math.exp(-v))


def test_expert_onehot_hidden_intermediate_closed_form():
    rng = np.random.default_rng(1)
    H, I = 256, 128
    h0, i0 = 77, 5
    w13 = np.zeros((1, 2 * I, H), np.float32)
    w13[0, i0, h0] = 1.0  # gate row i0 sees x[h0]
    w13[0, I + i0, h0] = 1.0  # up row i0 sees x[h0]
    w2 = (rng.standard_normal((1, H, I)) * 0.05).astype(np.float32)
    w13b, w2b = bf16(w13), bf16(w2)
    x = np.zeros((1, H))
    x[0, h0] = 1.0
    y = oracle.expert_rows("bf16", "bf16", w13b, None, w2b, None, 0, I, H, x)
    want = oracle.bf16_value(w2b[0, :, i0]) * silu(1.0)
    assert np.allclose(y[0], want, rtol=1e-15, atol=0)
    # transposing either operand would move the signal: check a different column is silent
    assert np.abs(y[0]).max() > 0


def test_expert_onehot_input_picks_weight_column():
    rng = np.random.default_rng(2)
    H, I = 128, 128
    w13 = bf16(rng.standard_normal((1, 2 * I, H)) * 0.3)
    w2 = bf16(rng.standard_normal((1, H, I)) * 0.3)
    W13 = oracle.bf16_value(w13)[0]
    W2 = oracle.bf16_value(w2)[0]
    for h0 in (0, 63, 127):
        x = np.zeros((1, H))
        x[0, h0] = 2.0
        y = oracle.expert_rows("bf16", "bf16", w13, None, w2, None, 0, I, H, x)
        g = 2.0 * W13[:I, h0]
        u = 2.0 * W13[I:, h0]
        a = g / (1 + np.exp(-g)) * u
        assert np.allclose(y[0], W2 @ a, rtol=1e-12, atol=1e-15)


def test_expert_zero_gate_gives_zero():
    rng = np.random.default_rng(3)
    H, I = 128, 128
    w13 = rng.standard_normal((1, 2 * I, H)).astype(np.float32)
    w13[0, :I] = 0.0
    w2 = rng.standard_normal((1, H, I)).astype(np.float32)
    x = rng.standard_normal((3, H))
    y = oracle.expert_rows("bf16", "bf16", bf16(w13), None, bf16(w2), None, 0, I, H, x)
    assert np.all(y == 0.0)


def test_expert_linear_in_down_projection_and_selects_matrix():
    rng = np.random.default_rng(4)
    H, I = 128, 256
    w13 = bf16(rng.standard_normal((3, 2 * I, H)) * 0.1)
    w2 = rng.standard_normal((3, H, I)).astype(np.float32) * 0.1
    w2b = bf16(w2)
    w2b2 = bf16(oracle.bf16_value(w2b) * 2.0)  # exact doubling in bf16
    x = rng.standard_normal((2, H))
    y1 = oracle.expert_rows("bf16", "bf16", w13, None, w2b, None, 2, I, H, x)
    y2 = oracle.expert_rows("bf16", "bf16", w13, None, w2b2, None, 2, I, H, x)
    assert np.array_equal(y2, 2.0 * y1)
    # matrix 2 of the stacked tensor equals matrix 0 of its own slice
    y3 = oracle.expert_rows("bf16", "bf16", w13[2:3], None, w2b[2:3], None, 0, I, H, x)
    assert np.array_equal(y1, y3)
    y0 = oracle.expert_rows("bf16", "bf16", w13, None, w2b, None, 0, I, H, x)
    assert not np.allclose(y0, y1)


def test_expert_fp8_scale_is_applied_per_block():
    rng = np.random.default_rng(5)
    H, I = 256, 128
    codes13 = rng.integers(0, 0x7E, (1, 2 * I, H), dtype=np.uint8)
    codes2 = rng.integers(0, 0x7E, (1, H, I), dtype=np.uint8)
    s13 = np.full((1, 2 * I // 128, H // 128), 0.5, np.float32)
    s2 = np.full((1, H // 128, I // 128), 0.25, np.float32)
    x = rng.standard_normal((1, H)) * 0.01
    y = oracle.expert_rows("fp8_e4m3_b128x128", "bf16", codes13, s13, codes2, s2, 0, I, H, x)
    W13 = oracle.e4m3_value(codes13)[0] * 0.5
    W2 = oracle.e4m3_value(codes2)[0] * 0.25
    g, u = W13[:I] @ x[0], W13[I:] @ x[0]
    assert np.allclose(y[0], W2 @ (g / (1 + np.exp(-g)) * u), rtol=1e-10, atol=1e-14)
    # scaling only the second hidden block of w13 by 2 changes the result (block placement)
    s13b = s13.copy()
    s13b[0, :, 1] = 1.0
    y2 = oracle.expert_rows("fp8_e4m3_b128x128", "bf16", codes13, s13b, codes2, s2, 0, I, H, x)
    assert not np.allclose(y, y2)


def test_expert_input_quantises_each_row():
    rng = np.random.default_rng(6)
    x = bf16(rng.standard_normal((3, 256)) * 3)
    for afmt in ("fp8_e4m3_pow2_b128", "mxfp8"):
        xin, q, sc = oracle.expert_input(afmt, x)
        for r in range(3):
            qq, ss = oracle.quant_act(afmt, oracle.bf16_value(x[r]))
            assert np.array_equal(q[r], qq) and np.array_equal(sc[r], ss)
            assert np.array_equal(xin[r], oracle.dequant_act(afmt, qq, ss))
    xin, q, sc = oracle.expert_input("bf16", x)
    assert q is None and np.array_equal(xin, oracle.bf16_value(x))


# ----------------------------------------------------------------- layer
def small_cfg(**kw):
    base = dict(hidden=128, n_routed_experts=8, num_experts_per_tok=3, n_group=1, topk_group=1,
                moe_intermediate_size=128, n_shared_experts=1, shared_intermediate_size=128,
                norm_topk_prob=True, routed_scaling_factor=2.827, score_fn="sigmoid", wfmt="bf16",
                afmt="bf16")
    base.update(kw)
    return SimpleNamespace(**base)


def test_layer_identical_experts_reduce_to_rsf_times_one_expert():
    rng = np.random.default_rng(7)
    c = small_cfg(n_shared_experts=2)
    H, I = c.hidden, c.moe_intermediate_size
    w13 = bf16(rng.standard_normal((1, 2 * I, H)) * 0.1)
    w2 = bf16(rng.standard_normal((1, H, I)) * 0.1)
    s13 = bf16(rng.standard_normal((2, 2 * I, H)) * 0.1)
    s2 = bf16(rng.standard_normal((2, H, I)) * 0.1)
    x = bf16(rng.standard_normal((5, H)))
    wg = (rng.standard_normal((c.n_routed_experts, H)) * 0.1).astype(np.float32)
    r = oracle.route(c, x, wg, np.zeros(c.n_routed_experts, np.float32))
    out = oracle.layer(c, x, r["idx"], r["w"], lambda e: (w13, None, w2, None),
                       lambda s: (s13[s:s + 1], None, s2[s:s + 1], None))
    xin = oracle.bf16_value(x)
    y = oracle.expert_rows("bf16", "bf16", w13, None, w2, None, 0, I, H, xin)
    sh = sum(oracle.expert_rows("bf16", "bf16", s13, None, s2, None, s, I, H, xin) for s in range(2))
    assert np.allclose(out, c.routed_scaling_factor * y + sh, rtol=1e-12, atol=1e-14)


def test_layer_zero_shared_and_weighted_sum():
    rng = np.random.default_rng(8)
    c = small_cfg()
    H, I, E = c.hidden, c.moe_intermediate_size, c.n_routed_experts
    w13 = bf16(rng.standard_normal((E, 2 * I, H)) * 0.1)
    w2 = bf16(rng.standard_normal((E, H, I)) * 0.1)
    zeros13 = bf16(np.zeros((1, 2 * I, H)))
    zeros2 = bf16(np.zeros((1, H, I)))
    x = bf16(rng.standard_normal((4, H)))
    idx = np.array([[0, 1, 2], [7, 6, 5], [3, 0, 7], [1, 2, 3]], np.int32)
    w = rng.uniform(0.1, 1.0, (4, 3))
    out = oracle.layer(c, x, idx, w, lambda e: (w13[e:e + 1], None, w2[e:e + 1], None),
                       lambda s: (zeros13, None, zeros2, None))
    xin = oracle.bf16_value(x)
    for t in range(4):
        want = sum(w[t, j] * oracle.expert_rows("bf16", "bf16", w13, None, w2, None, int(idx[t, j]),
                                                I, H, xin[t:t + 1])[0] for j in range(3))
        assert np.allclose(out[t], want, rtol=1e-12, atol=1e-15)


def test_swiglu_limit_closed_forms():
    """One-hot input rows make g and u equal to chosen weight columns, so the
    clamped SwiGLU has closed forms: min(g, L) for the gate, clamp(u, -L, L) for
    the up projection; a limit above every |g|, |u| changes nothing."""
    H, I, L = 8, 4, 0.5
    g = np.array([2.0, -3.0, 0.25, -0.5], np.float32)
    u = np.array([1.0, -2.0, 0.125, 4.0], np.float32)
    w13 = np.zeros((1, 2 * I, H), np.float32)
    w13[0, :I, 0] = g
    w13[0, I:, 0] = u
    w2 = np.zeros((1, H, I), np.float32)
    w2[0, np.arange(I), np.arange(I)] = 1.0  # y_i = a_i for i < I
    x = np.zeros((1, H))
    x[0, 0] = 1.0

    def silu(z):
        return z / (1.0 + math.exp(-z))

    y = oracle.expert_rows("bf16", "bf16", bf16(w13), None, bf16(w2), None, 0, I, H, x, limit=L)
    want = [silu(min(float(gi), L)) * max(min(float(ui), L), -L) for gi, ui in zip(g, u)]
    assert np.allclose(y[0, :I], want, rtol=1e-15, atol=0)
    y_off = oracle.expert_rows("bf16", "bf16", bf16(w13), None, bf16(w2), None, 0, I, H, x)
    y_big = oracle.expert_rows("bf16", "bf16", bf16(w13), None, bf16(w2), None, 0, I, H, x,
                               limit=10.0)
    assert np.array_equal(y_off, y_big)
    assert np.allclose(y_off[0, :I], [silu(float(gi)) * float(ui) for gi, ui in zip(g, u)],
                       rtol=1e-15)
