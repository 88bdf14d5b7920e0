"""Pins of the oracle's composed layer (routing, experts and combine together)
by properties the layer's definition fixes for any weights: each token's output
depends on that token alone, relabelling the experts (router rows, biases and
expert weights together) changes nothing, the routed part scales exactly with
routed_scaling_factor, and a constant added to every bias leaves the selection
and the weights unchanged ("DeepSeek V3架构拆解：Kimi-K2-Thinking-NVFP4的MLA注意力与MoE
路由实现原理", 三.1–三.4). A wrong token, slot or expert index anywhere in the
composition breaks one of them."""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def cfg(**kw):
    base = dict(hidden=128, n_routed_experts=12, num_experts_per_tok=3, n_group=1, topk_group=1,
                moe_intermediate_size=64, n_shared_experts=1, shared_intermediate_size=64,
                norm_topk_prob=True, routed_scaling_factor=2.5, score_fn="sigmoid", wfmt="bf16",
                afmt="bf16")
    base.update(kw)
    return SimpleNamespace(**base)


def model(c, seed, zero_shared=False):
    rng = np.random.default_rng(seed)
    H, I, E, S = c.hidden, c.moe_intermediate_size, c.n_routed_experts, c.n_shared_experts
    m = {
        "wg": (rng.standard_normal((E, H)) * 0.1).astype(np.float32),
        "bias": rng.uniform(-0.1, 0.1, E).astype(np.float32),
        "w13": bf16(rng.standard_normal((E, 2 * I, H)) * 0.1),
        "w2": bf16(rng.standard_normal((E, H, I)) * 0.1),
        "s13": bf16(rng.standard_normal((S, 2 * c.shared_intermediate_size, H)) * 0.1),
        "s2": bf16(rng.standard_normal((S, H, c.shared_intermediate_size)) * 0.1),
    }
    if zero_shared:
        m["s13"] = bf16(np.zeros_like(m["s13"], dtype=np.float32))
        m["s2"] = bf16(np.zeros_like(m["s2"], dtype=np.float32))
    return m


def run(c, m, x):
    r = oracle.route(c, x, m["wg"], m["bias"])
    out = oracle.layer(c, x, r["idx"], r["w"],
                       lambda e: (m["w13"][e:e + 1], None, m["w2"][e:e + 1], None),
                       lambda s: (m["s13"][s:s + 1], None, m["s2"][s:s + 1], None))
    return r, out


CFGS = [cfg(), cfg(score_fn="sqrtsoftplus", norm_topk_prob=False),
        cfg(n_group=4, topk_group=2), cfg(afmt="fp8_e4m3_pow2_b128", score_fn="softmax", moe_intermediate_size=128,
            shared_intermediate_size=128),
        cfg(afmt="mxfp8", n_shared_experts=2)]


@pytest.mark.parametrize("c", CFGS, ids=["sigmoid", "sqrtsoftplus", "grouped", "fp8act", "mxfp8"])
def test_each_token_depends_on_itself_alone(c):
    """Reordering, duplicating and dropping tokens reorders, duplicates and drops
    output rows, bit for bit."""
    m = model(c, 11)
    rng = np.random.default_rng(12)
    x = bf16(rng.standard_normal((9, c.hidden)))
    _, out = run(c, m, x)
    perm = np.array([4, 0, 8, 8, 2, 7, 1])  # reordered, token 8 twice, tokens 3, 5, 6 absent
    _, out_p = run(c, m, x[perm])
    assert np.array_equal(out_p, out[perm])


@pytest.mark.parametrize("c", CFGS[:3], ids=["sigmoid", "sqrtsoftplus", "grouped"])
def test_relabelling_experts_changes_nothing(c):
    """Experts relabelled by a permutation that keeps each group's members in that
    group (router rows, biases and expert weights moved together): the same
    experts are chosen, under their new ids, and the output is unchanged."""
    m = model(c, 21)
    E, G = c.n_routed_experts, c.n_group
    gs = E // G
    rng = np.random.default_rng(22)
    # new id of old expert e: shuffle inside each group, then shuffle whole groups
    gperm = rng.permutation(G)
    new_of = np.empty(E, np.int64)
    for g in range(G):
        members = rng.permutation(gs)
        new_of[g * gs:(g + 1) * gs] = gperm[g] * gs + members
    old_of = np.argsort(new_of)
    m2 = dict(m)
    for key in ("wg", "bias", "w13", "w2"):
        m2[key] = np.ascontiguousarray(m[key][old_of])
    x = bf16(rng.standard_normal((8, c.hidden)))
    r, out = run(c, m, x)
    r2, out2 = run(c, m2, x)
    assert not r["near_tie"].any() and not r2["near_tie"].any()
    for t in range(x.shape[0]):
        # same set of experts with the same weights (slot order may differ only on ties)
        a = sorted(zip(new_of[r["idx"][t]].tolist(), r["w"][t].tolist()))
        b = sorted(zip(r2["idx"][t].tolist(), r2["w"][t].tolist()))
        assert a == b
    assert np.allclose(out2, out, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("norm", [True, False])
def test_routed_part_scales_exactly_with_the_scaling_factor(norm):
    """With the shared expert's weights zero, the output is the routed sum alone,
    and doubling routed_scaling_factor doubles it exactly (a power of two)."""
    c1 = cfg(norm_topk_prob=norm, routed_scaling_factor=1.25)
    c2 = cfg(norm_topk_prob=norm, routed_scaling_factor=2.5)
    m = model(c1, 31, zero_shared=True)
    x = bf16(np.random.default_rng(32).standard_normal((6, c1.hidden)))
    r1, out1 = run(c1, m, x)
    r2, out2 = run(c2, m, x)
    assert np.array_equal(r1["idx"], r2["idx"])
    assert np.array_equal(r2["w"], 2.0 * r1["w"])
    assert np.array_equal(out2, 2.0 * out1)
    assert np.any(out1 != 0.0)


@pytest.mark.parametrize("c", CFGS[:3], ids=["sigmoid", "sqrtsoftplus", "grouped"])
def test_a_common_bias_shift_changes_nothing(c):
    """Adding one constant to every expert's bias shifts every biased score (and
    every group score) alike, so the selection is the same, and the weights come
    from the unbiased scores, so they are the same too."""
    m = model(c, 41)
    m2 = dict(m)
    m2["bias"] = (m["bias"] + np.float32(0.5)).astype(np.float32)
    x = bf16(np.random.default_rng(42).standard_normal((8, c.hidden)))
    r, out = run(c, m, x)
    r2, out2 = run(c, m2, x)
    ok = ~(r["near_tie"] | r2["near_tie"])
    assert ok.sum() >= 6
    assert np.array_equal(r["idx"][ok], r2["idx"][ok])
    assert np.array_equal(r["w"][ok], r2["w"][ok])
    assert np.array_equal(out[ok], out2[ok])


# ----------------------------------------------------------------- planted mistakes
def test_a_row_mixup_in_the_experts_breaks_token_locality(monkeypatch):
    """Planted in the oracle: each expert gets its rows rotated by one (a wrong
    token index). The token-locality property no longer holds."""
    c = cfg()
    m = model(c, 11)
    x = bf16(np.random.default_rng(12).standard_normal((9, c.hidden)))
    real = oracle.expert_rows

    def rotated(wfmt, afmt, w13, w13s, w2, w2s, e, I, H, xin, limit=0.0):
        return real(wfmt, afmt, w13, w13s, w2, w2s, e, I, H, np.roll(xin, 1, axis=0), limit)

    monkeypatch.setattr(oracle, "expert_rows", rotated)
    _, out = run(c, m, x)
    perm = np.array([4, 0, 8, 8, 2, 7, 1])
    _, out_p = run(c, m, x[perm])
    assert not np.array_equal(out_p, out[perm])


def test_an_expert_off_by_one_breaks_relabelling():
    """Planted in the caller of the oracle: expert e runs with expert e+1's
    weights. The relabelled model then disagrees."""
    c = cfg()
    m = model(c, 21)
    E = c.n_routed_experts
    rng = np.random.default_rng(22)
    new_of = rng.permutation(E)
    old_of = np.argsort(new_of)
    m2 = dict(m)
    for key in ("wg", "bias", "w13", "w2"):
        m2[key] = np.ascontiguousarray(m[key][old_of])
    x = bf16(rng.standard_normal((8, c.hidden)))

    def run_off_by_one(mm):
        r = oracle.route(c, x, mm["wg"], mm["bias"])
        nxt = lambda e: (e + 1) % E
        return oracle.layer(c, x, r["idx"], r["w"],
                            lambda e: (mm["w13"][nxt(e):nxt(e) + 1], None,
                                       mm["w2"][nxt(e):nxt(e) + 1], None),
                            lambda s: (mm["s13"][s:s + 1], None, mm["s2"][s:s + 1], None))

    assert not np.allclose(run_off_by_one(m2), run_off_by_one(m), rtol=1e-6, atol=1e-9)
