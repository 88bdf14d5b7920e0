"""Pins of the oracle's router, scoring, group-limited top-k and weights:
brute-force enumeration on tiny expert counts, the n_group == 1 special case
against a library stable sort, closed forms of the scores, the stated weight
invariants, and constructed near-ties."""
import itertools
import math
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle


def cfg(E, k, ng=1, tg=1, H=8, norm=True, rsf=2.827, score="sigmoid"):
    return SimpleNamespace(hidden=H, n_routed_experts=E, num_experts_per_tok=k, n_group=ng,
                           topk_group=tg, moe_intermediate_size=128, n_shared_experts=0,
                           shared_intermediate_size=128, norm_topk_prob=norm,
                           routed_scaling_factor=rsf, score_fn=score, wfmt="bf16", afmt="bf16")


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def onehot_router(logits):
    """x = e_0 (bf16 1.0) and Wg[:, 0] = logits: the router returns the logits exactly."""
    E = len(logits)
    H = 8
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 1.0
    wg = np.zeros((E, H), np.float32)
    wg[:, 0] = logits
    return bf16(x), wg


def sigmoid(l):
    return 1.0 / (1.0 + np.exp(-np.asarray(l, np.float64)))


def test_router_logits_onehot_and_matmul():
    rng = np.random.default_rng(0)
    E, H = 12, 64
    wg = (rng.standard_normal((E, H)) * 0.1).astype(np.float32)
    c = cfg(E, 2, H=H)
    for h0 in (0, 17, 63):
        x = np.zeros(H, np.float32)
        x[h0] = 1.0
        r = oracle.route_token(c, bf16(x), wg, np.zeros(E, np.float32))
        assert np.array_equal(r["logits"], wg[:, h0].astype(np.float64))
    x = rng.standard_normal(H).astype(np.float32)
    xb = bf16(x)
    r = oracle.route_token(c, xb, wg, np.zeros(E, np.float32))
    ref = wg.astype(np.float64) @ oracle.bf16_value(xb)
    assert np.allclose(r["logits"], ref, rtol=0, atol=1e-13)


def test_score_closed_forms():
    assert oracle.score(0.0, "sigmoid") == 0.5
    for l in (-30.0, -2.5, 0.3, 7.0):
        assert abs(oracle.score(l, "sigmoid") + oracle.score(-l, "sigmoid") - 1.0) < 1e-15
    assert abs(oracle.score(0.0, "sqrtsoftplus") - math.sqrt(math.log(2.0))) < 1e-15
    for l in (20.0, 50.0, 700.0):
        assert abs(oracle.score(l, "sqrtsoftplus") - math.sqrt(l + math.log1p(math.exp(-l)))) < 1e-12
    assert oracle.score(800.0, "sqrtsoftplus") == pytest.approx(math.sqrt(800.0), rel=1e-15)
    v = oracle.score(-40.0, "sqrtsoftplus")
    assert v == pytest.approx(math.sqrt(math.log1p(math.exp(-40.0))), rel=1e-12)


def brute_force(sp, k, ng, tg):
    """Enumerate every group subset, then every k-subset of the kept experts."""
    E = len(sp)
    gsz = E // ng
    gscore = []
    for g in range(ng):
        vals = sorted(sp[g * gsz:(g + 1) * gsz], reverse=True)
        gscore.append(vals[0] if gsz == 1 else vals[0] + vals[1])
    best_groups = max(itertools.combinations(range(ng), tg), key=lambda s: sum(gscore[g] for g in s))
    cand = [e for e in range(E) if e // gsz in best_groups]
    best = max(itertools.combinations(cand, k), key=lambda s: sum(sp[e] for e in s))
    return set(best)


@pytest.mark.parametrize("E,k,ng,tg", [(8, 2, 1, 1), (8, 3, 4, 2), (12, 4, 3, 2), (12, 2, 6, 3),
                                       (16, 4, 4, 2), (16, 3, 8, 4), (16, 4, 16, 4), (10, 10, 1, 1),
                                       (16, 5, 2, 1)])
def test_group_topk_matches_brute_force(E, k, ng, tg):
    rng = np.random.default_rng(E * 100 + k * 10 + ng)
    c = cfg(E, k, ng, tg)
    for trial in range(40):
        logits = rng.standard_normal(E).astype(np.float32)
        bias = (rng.uniform(-0.2, 0.2, E)).astype(np.float32)
        x, wg = onehot_router(logits)
        r = oracle.route_token(c, x, wg, bias)
        sp = sigmoid(logits) + bias.astype(np.float64)
        assert set(r["idx"].tolist()) == brute_force(sp, k, ng, tg)
        # slot order: biased score descending
        assert np.all(np.diff(sp[r["idx"]]) <= 0)


def test_single_group_is_plain_topk():
    rng = np.random.default_rng(1)
    E, k = 384, 8
    c = cfg(E, k)
    for trial in range(20):
        logits = (rng.standard_normal(E) * 1.7).astype(np.float32)
        bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
        x, wg = onehot_router(logits)
        r = oracle.route_token(c, x, wg, bias)
        sp = sigmoid(logits) + bias.astype(np.float64)
        ref = np.argsort(-sp, kind="stable")[:k]
        assert np.array_equal(r["idx"], ref)
        ref_t = torch.topk(torch.from_numpy(sp), k).indices.numpy()
        assert np.array_equal(r["idx"], ref_t)


def test_ties_go_to_lower_index():
    E, k = 16, 4
    x, wg = onehot_router(np.zeros(E, np.float32))
    r = oracle.route_token(cfg(E, k), x, wg, np.zeros(E, np.float32))
    assert r["idx"].tolist() == [0, 1, 2, 3]
    assert r["near_tie"]
    # all-equal groups: the lower groups are kept
    r = oracle.route_token(cfg(E, k, 4, 2), x, wg, np.zeros(E, np.float32))
    assert r["idx"].tolist() == [0, 1, 2, 3]


def test_weights_normalised_unbiased_and_scaled():
    rng = np.random.default_rng(2)
    E, k, rsf = 32, 6, 2.827
    for norm in (True, False):
        c = cfg(E, k, norm=norm, rsf=rsf)
        for trial in range(20):
            logits = rng.standard_normal(E).astype(np.float32)
            bias = rng.uniform(-0.3, 0.3, E).astype(np.float32)
            x, wg = onehot_router(logits)
            r = oracle.route_token(c, x, wg, bias)
            s = sigmoid(logits)
            if norm:
                assert abs(r["w"].sum() - rsf) < 1e-12
                assert np.all(r["w"] > 0) and np.all(r["w"] <= rsf)
                assert np.allclose(r["w"] / rsf * s[r["idx"]].sum(), s[r["idx"]], rtol=1e-14)
            else:
                assert np.allclose(r["w"], s[r["idx"]] * rsf, rtol=1e-15)


def test_bias_steers_selection_but_not_weights():
    E, k = 8, 2
    logits = np.array([3.0, 2.0, 1.0, 0.0, -1.0, -2.0, -3.0, -4.0], np.float32)
    bias = np.zeros(E, np.float32)
    bias[7] = 1.0  # sigmoid(-4) + 1 beats everything
    x, wg = onehot_router(logits)
    r = oracle.route_token(cfg(E, k, rsf=1.0), x, wg, bias)
    assert r["idx"].tolist() == [7, 0]
    s = sigmoid(logits)
    assert np.allclose(r["w"], [s[7] / (s[7] + s[0]), s[0] / (s[7] + s[0])], rtol=1e-15)


def test_sqrtsoftplus_routing():
    rng = np.random.default_rng(3)
    E, k = 64, 6
    c = cfg(E, k, rsf=2.5, score="sqrtsoftplus")
    logits = rng.standard_normal(E).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    x, wg = onehot_router(logits)
    r = oracle.route_token(c, x, wg, bias)
    l = logits.astype(np.float64)
    s = np.sqrt(np.log1p(np.exp(l)))
    assert np.array_equal(r["idx"], np.argsort(-(s + bias), kind="stable")[:k])
    assert np.allclose(r["w"], s[r["idx"]] / s[r["idx"]].sum() * 2.5, rtol=1e-14)


def test_near_tie_reported():
    E, k = 8, 2
    logits = np.array([2.0, 1.0, 0.5, 0.0, -1, -1, -1, -1], np.float32)
    s = sigmoid(logits)
    bias = np.zeros(E, np.float64)
    bias[2] = s[1] - s[2] + 1e-9  # expert 2 sits 1e-9 above expert 1 at the k boundary
    x, wg = onehot_router(logits)
    r = oracle.route_token(cfg(E, k), x, wg, bias.astype(np.float32))
    # float32 bias cannot carry 1e-9 exactly; the gap is tiny either way
    assert r["near_tie"] and r["gap"] < 1e-6
    r = oracle.route_token(cfg(E, k), x, wg, np.zeros(E, np.float32))
    assert not r["near_tie"] and r["gap"] > 1e-3


def test_slot_order_near_tie_reported():
    """Two chosen experts whose biased scores sit within 1e-6 (relative) of each
    other make the slot order a near-tie, not the set: the order gap is the
    smallest relative gap between consecutive slots, by brute force over the
    constructed scores."""
    E, k = 8, 3
    logits = np.zeros(E, np.float32)  # s = 0.5 everywhere
    bias = np.array([0.30, 0.20, 0.20, 0.10, 0.0, -0.1, -0.2, -0.3], np.float32)
    bias[2] = np.nextafter(np.float32(0.20), np.float32(1.0))  # one float32 ulp above expert 1
    x, wg = onehot_router(logits)
    r = oracle.route_token(cfg(E, k), x, wg, bias)
    assert r["idx"].tolist() == [0, 2, 1]
    sp = 0.5 + bias.astype(np.float64)
    want = min(abs(sp[a] - sp[b]) / max(abs(sp[a]), abs(sp[b]))
               for a, b in ((0, 2), (2, 1)))
    assert r["order_gap"] == want and r["order_tie"]
    assert not r["near_tie"]  # the k-th and (k+1)-th are 0.1 apart
    many = oracle.route(cfg(E, k), x, wg, bias)
    assert many["order_tie"][0] and many["order_gap"][0] == want
    # well separated slots: no order near-tie; k = 1 has no consecutive pair
    r = oracle.route_token(cfg(E, k), x, wg, np.array([0.3, 0.2, 0.1, 0, -0.1, -0.2, -0.3, -0.4],
                                                      np.float32))
    assert not r["order_tie"] and r["order_gap"] > 0.1
    r = oracle.route_token(cfg(E, 1), x, wg, bias)
    assert r["order_gap"] == math.inf


def test_group_near_tie_reported():
    E, k, ng, tg = 8, 2, 4, 2
    # groups of 2: group sums 2s, with groups 1 and 2 equal -> tie at the kept/dropped boundary
    logits = np.array([3.0, 3.0, 1.0, 1.0, 1.0, 1.0, -2.0, -2.0], np.float32)
    x, wg = onehot_router(logits)
    r = oracle.route_token(cfg(E, k, ng, tg), x, wg, np.zeros(E, np.float32))
    assert r["near_tie"]
    assert set(r["idx"].tolist()) == {0, 1}


def test_group_of_one_and_k_equals_E():
    rng = np.random.default_rng(4)
    E = 16
    logits = rng.standard_normal(E).astype(np.float32)
    x, wg = onehot_router(logits)
    s = sigmoid(logits)
    r = oracle.route_token(cfg(E, 3, ng=E, tg=5), x, wg, np.zeros(E, np.float32))
    assert np.array_equal(r["idx"], np.argsort(-s, kind="stable")[:3])
    r = oracle.route_token(cfg(E, E), x, wg, np.zeros(E, np.float32))
    assert sorted(r["idx"].tolist()) == list(range(E))


def test_too_few_candidates_is_an_error():
    E = 8
    x, wg = onehot_router(np.zeros(E, np.float32))
    with pytest.raises(ValueError):
        oracle.route_token(cfg(E, 5, ng=4, tg=2), x, wg, np.zeros(E, np.float32))


def test_route_many_tokens_equals_per_token():
    rng = np.random.default_rng(5)
    E, k, H, T = 24, 4, 64, 50
    c = cfg(E, k, ng=4, tg=2, H=H)
    x = bf16(rng.standard_normal((T, H)))
    wg = (rng.standard_normal((E, H)) * 0.1).astype(np.float32)
    b = rng.uniform(-0.05, 0.05, E).astype(np.float32)
    r = oracle.route(c, x, wg, b)
    toks = np.array([3, 49, 0], np.int32)
    rs = oracle.route(c, x, wg, b, tokens=toks)
    for i, t in enumerate(toks):
        one = oracle.route_token(c, x[t], wg, b)
        assert np.array_equal(r["idx"][t], one["idx"]) and np.array_equal(rs["idx"][i], one["idx"])
        assert np.array_equal(r["w"][t], one["w"])
    # each token picks k distinct experts
    assert all(len(set(row)) == k for row in r["idx"].tolist())


# ----------------------------------------------------------------- softmax scoring
def test_softmax_equal_logits_give_uniform_scores():
    """All logits equal: every expert scores 1/E; ties go to the lower indices,
    and the unnormalised weights are rsf/E each."""
    E, k = 16, 4
    c = cfg(E, k, norm=False, rsf=1.5, score="softmax")
    x, wg = onehot_router(np.full(E, 0.75, np.float32))
    r = oracle.route_token(c, x, wg, np.zeros(E, np.float32))
    assert list(r["idx"]) == [0, 1, 2, 3]
    assert np.allclose(r["w"], 1.5 / E, rtol=1e-15)


def test_softmax_scores_sum_to_one_and_follow_exp_ratios():
    """k = E without normalisation returns every probability: they sum to rsf,
    and any two are in the ratio exp(l_i - l_j) (the property that defines
    softmax); adding a constant to all logits changes nothing."""
    rng = np.random.default_rng(11)
    E = 32
    c = cfg(E, E, norm=False, rsf=2.0, score="softmax")
    # on a 2^-10 grid, so adding 40 below is exact in float32
    logits = (np.round(rng.standard_normal(E) * 3 * 1024) / 1024).astype(np.float32)
    x, wg = onehot_router(logits)
    r = oracle.route_token(c, x, wg, np.zeros(E, np.float32))
    w = r["w"] / 2.0
    assert abs(w.sum() - 1.0) < 1e-14
    l = logits.astype(np.float64)[r["idx"]]
    for i in range(E):
        assert math.isclose(w[i] / w[0], math.exp(l[i] - l[0]), rel_tol=1e-12)
    x2, wg2 = onehot_router(logits + np.float32(40.0))  # large shift: exp would overflow unshifted
    r2 = oracle.route_token(c, x2, wg2, np.zeros(E, np.float32))
    assert np.array_equal(r["idx"], r2["idx"]) and np.allclose(r["w"], r2["w"], rtol=1e-12)


@pytest.mark.parametrize("ng,tg", [(1, 1), (4, 2)])
def test_softmax_selection_is_brute_force_topk_of_biased_scores(ng, tg):
    """Selection on softmax + bias matches exhaustive search over expert subsets
    of the kept groups (softmax is monotone in the logit, but the bias is added
    to the probability, so the order can differ from the logits' order)."""
    rng = np.random.default_rng(12 + ng)
    E, k = 8, 3
    c = cfg(E, k, ng=ng, tg=tg, score="softmax")
    logits = rng.standard_normal(E).astype(np.float32)
    bias = rng.uniform(-0.2, 0.2, E).astype(np.float32)
    x, wg = onehot_router(logits)
    r = oracle.route_token(c, x, wg, bias)
    l = logits.astype(np.float64)
    p = np.exp(l - l.max())
    p /= p.sum()
    sp = p + bias
    gsz = E // ng
    gs = [sum(sorted(sp[g * gsz:(g + 1) * gsz])[-2:]) for g in range(ng)]
    kept = sorted(range(ng), key=lambda g: -gs[g])[:tg] if ng > 1 else [0]
    cand = [e for e in range(E) if e // gsz in kept]
    best = max(itertools.combinations(cand, k), key=lambda sub: sum(sp[e] for e in sub))
    assert sorted(r["idx"]) == sorted(best)
    assert np.allclose(r["w"], p[r["idx"]] / p[r["idx"]].sum() * c.routed_scaling_factor, rtol=1e-12)
