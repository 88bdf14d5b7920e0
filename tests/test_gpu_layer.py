"""GPU parity of the whole layer and its steps against the float64 oracle, on
the seeded workloads, through the C ABI."""
import numpy as np
import pytest
import torch

import expert_routing_grouped_layer_b200 as moe
import oracle
from expert_routing_grouped_layer_b200 import workloads as W
from moe_testlib import (LAYER_TOL, check_layer_tokens, check_permutation_properties,
                         compare_permutation_exact, compare_routing, gpu_forward, oracle_route)

pytestmark = pytest.mark.gpu


def _data(cfg):
    inp = W.make_inputs(cfg, "cuda")
    wts = W.make_weights(cfg, "cuda")
    return inp, wts


def _full_check(cfg, inp, wts, T=None):
    """Routing of every token (sets and weights, near-ties excepted), the
    permutation element by element, and every token's output against the oracle."""
    T = cfg.T if T is None else T
    g = gpu_forward(cfg, inp, wts, T)
    assert g["status"] == 0
    r = oracle_route(cfg, inp, T=T)
    compare_routing(cfg, g, r, np.arange(T))
    check_permutation_properties(cfg, g, T)
    compare_permutation_exact(cfg, g, r)
    toks = np.nonzero(~r["near_tie"])[0]
    err = check_layer_tokens(cfg, inp, wts, g, r, toks, LAYER_TOL[cfg.afmt])
    return g, r, float(err.max())


def test_tiny_layer_full_parity():
    cfg = W.CONFIGS["tiny_bf16"]
    inp, wts = _data(cfg)
    g, r, err = _full_check(cfg, inp, wts)
    assert np.array_equal(g["idx"], r["idx"])  # slot order too
    assert (np.abs(g["w"] - r["w"]) <= 1e-5 * np.abs(r["w"])).all()


@pytest.mark.parametrize("T", [1, 5, 17, 37, 63])
def test_tiny_layer_ragged_token_counts(T):
    cfg = W.CONFIGS["tiny_bf16"]
    inp, wts = _data(cfg)
    _full_check(cfg, inp, wts, T=T)


def test_tiny_one_expert_takes_every_token():
    cfg = W.CONFIGS["tiny_bf16"]
    inp, wts = _data(cfg)
    inp["gate_bias"][5] = 10.0  # expert 5 wins every token's first slot
    g, r, _ = _full_check(cfg, inp, wts)
    assert (g["idx"][:, 0] == 5).all()
    assert g["offsets"][6] - g["offsets"][5] == cfg.T


def test_tiny_all_equal_scores_tie_break():
    cfg = W.CONFIGS["tiny_bf16"]
    inp, wts = _data(cfg)
    inp["gate_w"].zero_()
    inp["gate_bias"].zero_()
    g = gpu_forward(cfg, inp, wts)
    assert (g["idx"] == np.arange(cfg.num_experts_per_tok)).all()
    np.testing.assert_allclose(g["w"], cfg.routed_scaling_factor / cfg.num_experts_per_tok,
                               rtol=1e-6)
    check_permutation_properties(cfg, g)
    # experts >= k receive nothing: the empty blocks are skipped
    assert (np.diff(g["offsets"])[cfg.num_experts_per_tok:] == 0).all()


@pytest.mark.parametrize("ng,tg,k", [(4, 2, 4), (16, 4, 4), (8, 8, 6), (2, 1, 8)])
def test_tiny_group_limited(ng, tg, k):
    cfg = W.CONFIGS["tiny_bf16"].replace(n_group=ng, topk_group=tg, num_experts_per_tok=k)
    inp, wts = _data(cfg)
    _full_check(cfg, inp, wts)


def test_tiny_k_equals_E_and_no_norm_and_sqrtsoftplus():
    base = W.CONFIGS["tiny_bf16"]
    for cfg in (base.replace(num_experts_per_tok=16),
                base.replace(norm_topk_prob=False),
                base.replace(score_fn="sqrtsoftplus", routed_scaling_factor=2.5),
                base.replace(n_shared_experts=0),
                base.replace(n_shared_experts=2)):
        inp, wts = _data(cfg)
        _full_check(cfg, inp, wts)


def test_tiny_larger_shapes_span_tiles():
    # several M tiles (H = 512 -> 4 down-projection tiles), several K blocks,
    # several token tiles per expert (T*k/E > 128) and a ragged last tile
    cfg = W.CONFIGS["tiny_bf16"].replace(T=700, hidden=512, moe_intermediate_size=256,
                                         shared_intermediate_size=256, n_routed_experts=8,
                                         num_experts_per_tok=3)
    inp, wts = _data(cfg)
    _full_check(cfg, inp, wts)


def test_decode_bf16_full_size():
    """The decode layer at full size: routing of all 128 tokens, the permutation
    element by element, and the output of every token against the oracle."""
    cfg = W.CONFIGS["k2_decode_bf16"]
    inp, wts = _data(cfg)
    g = gpu_forward(cfg, inp, wts)
    assert g["status"] == 0
    r = oracle_route(cfg, inp)  # routing of every token
    compare_routing(cfg, g, r, np.arange(cfg.T))
    check_permutation_properties(cfg, g)
    compare_permutation_exact(cfg, g, r)
    active = int((np.diff(g["offsets"]) > 0).sum())
    assert 100 <= active <= 384
    toks = np.nonzero(~r["near_tie"])[0]
    check_layer_tokens(cfg, inp, wts, g, r, toks, LAYER_TOL["bf16"])


def test_step_entry_points_match_layer():
    """moe_gate_topk -> moe_permute -> moe_grouped_swiglu -> moe_combine called
    one by one equal moe_layer_forward bit for bit."""
    cfg = W.CONFIGS["tiny_bf16"]
    inp, wts = _data(cfg)
    T, k, E, H = cfg.T, cfg.num_experts_per_tok, cfg.n_routed_experts, cfg.hidden
    ws = torch.empty(moe.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_gate_topk(cfg, inp["x"], T, inp["gate_w"], inp["gate_bias"], idx, tw, ws, st)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ro = torch.empty(T * k, dtype=torch.int32, device="cuda")
    moe.moe_permute(cfg, idx, T, off, sp, ro, st, ws)
    y = torch.empty(T * k, H, dtype=torch.bfloat16, device="cuda")
    sy = torch.empty(cfg.n_shared_experts, T, H, dtype=torch.bfloat16, device="cuda")
    w = dict(wts)
    moe.moe_grouped_swiglu(cfg, inp["x"], T, sp, off, w, y, sy, ws, st)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(cfg, y, sy, ro, tw, T, out)
    torch.cuda.synchronize()
    g = gpu_forward(cfg, inp, wts)
    assert st.item() == 0
    assert np.array_equal(idx.cpu().numpy(), g["idx"])
    assert np.array_equal(out.float().cpu().numpy().astype(np.float64), g["out"])


def test_bad_expert_id_sets_status_and_is_skipped():
    cfg = W.CONFIGS["tiny_bf16"]
    T, k, E = 8, cfg.num_experts_per_tok, cfg.n_routed_experts
    idx = torch.arange(T * k, dtype=torch.int32, device="cuda").reshape(T, k) % E
    idx[3, 1] = E + 7
    idx[5, 0] = -2
    ws = torch.empty(moe.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.full((T * k,), -5, dtype=torch.int32, device="cuda")
    ro = torch.empty(T * k, dtype=torch.int32, device="cuda")
    moe.moe_permute(cfg, idx, T, off, sp, ro, st, ws)
    torch.cuda.synchronize()
    assert st.item() & moe.MOE_DEV_BAD_EXPERT
    ro = ro.cpu().numpy()
    assert ro[3 * k + 1] == -1 and ro[5 * k] == -1
    assert off.cpu().numpy()[E] == T * k - 2


@pytest.mark.parametrize("ng,tg,norm", [(1, 1, True), (4, 2, True), (1, 1, False)])
def test_tiny_softmax_scoring(ng, tg, norm):
    """Softmax over each token's logits instead of sigmoid: routing (sets, slot
    order, weights to 1e-5) and the layer output against the oracle."""
    cfg = W.CONFIGS["tiny_bf16"].replace(score_fn="softmax", n_group=ng, topk_group=tg,
                                         norm_topk_prob=norm)
    inp, wts = _data(cfg)
    g, r, _ = _full_check(cfg, inp, wts)
    ok = ~r["near_tie"]
    assert np.array_equal(g["idx"][ok], r["idx"][ok])
    assert (np.abs(g["w"][ok] - r["w"][ok]) <= 1e-5 * np.abs(r["w"][ok])).all()


@pytest.mark.parametrize("E,k", [(384, 8), (896, 16)])
def test_softmax_scoring_wide_expert_counts(E, k):
    """Softmax across 384 and 896 experts (12 and 28 scores per lane)."""
    cfg = W.CONFIGS["k2_decode_bf16"].replace(score_fn="softmax", T=64, hidden=512,
                                              moe_intermediate_size=256,
                                              shared_intermediate_size=256, n_routed_experts=E,
                                              num_experts_per_tok=k)
    inp, wts = _data(cfg)
    g, r, _ = _full_check(cfg, inp, wts)
    ok = ~r["near_tie"]
    assert (np.abs(g["w"][ok] - r["w"][ok]) <= 1e-5 * np.abs(r["w"][ok])).all()


_REORDER_CASES = {
    # several token tiles per expert with ragged ends, several M tiles
    "bf16": W.CONFIGS["tiny_bf16"].replace(T=700, hidden=512, moe_intermediate_size=256,
                                           shared_intermediate_size=256, n_routed_experts=8,
                                           num_experts_per_tok=3),
    "fp8w": W.CONFIGS["tiny_bf16"].replace(T=700, hidden=512, moe_intermediate_size=256,
                                           shared_intermediate_size=256, n_routed_experts=8,
                                           num_experts_per_tok=3, n_shared_experts=2,
                                           wfmt="fp8_e4m3_b128x128"),
    "fp4": W.CONFIGS["tiny_bf16"].replace(T=700, hidden=1024, moe_intermediate_size=512,
                                          shared_intermediate_size=512, n_routed_experts=8,
                                          num_experts_per_tok=3, wfmt="fp4_e2m1_ue8m0_b32",
                                          afmt="fp8_e4m3_pow2_b128", score_fn="sqrtsoftplus",
                                          routed_scaling_factor=2.5),
    "mx": W.CONFIGS["tiny_bf16"].replace(T=700, hidden=1024, moe_intermediate_size=512,
                                         shared_intermediate_size=512, n_routed_experts=8,
                                         num_experts_per_tok=3, wfmt="mxfp4", afmt="mxfp8",
                                         n_shared_experts=2),
    "decode_full": W.CONFIGS["k2_decode_bf16"],
}


@pytest.mark.parametrize("name", list(_REORDER_CASES))
def test_token_order_permutes_output_bit_for_bit(name):
    """Each token's output depends on that token alone ([V3] 三.4: every token is
    routed and combined on its own): at a fixed token count, feeding the tokens
    in another order must give the same rows in that order, bit for bit. The
    tokens land in other tiles and at other rows of them, so this checks that
    no kernel lets a row's arithmetic depend on its neighbours or its place."""
    cfg = _REORDER_CASES[name]
    inp, wts = _data(cfg)
    T = cfg.T
    layer = moe.MoELayer(cfg, wts, inp["gate_w"], inp["gate_bias"], max_tokens=T, device="cuda")
    out = layer.forward(inp["x"]).clone()
    g = torch.Generator(device="cpu").manual_seed(17)
    perm = torch.randperm(T, generator=g).to("cuda")
    out_p = layer.forward(inp["x"][perm].contiguous()).clone()
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    assert torch.equal(out_p.view(torch.int16), out[perm].view(torch.int16))
