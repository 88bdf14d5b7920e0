"""The synthetic workloads carry the pages' constants, and the weight encoder
writes valid codes (decoded here by the oracle's pinned decoders)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from expert_routing_grouped_layer_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def page():
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        return {k: v["value"] for k, v in json.load(f).items() if not k.startswith("_")}


def test_configs_carry_page_constants():
    p = page()
    for name in ("k2_decode_bf16", "k2_prefill_fp8w"):
        c = W.CONFIGS[name]
        assert c.n_routed_experts == p["k2_routed_experts"]
        assert c.n_shared_experts == p["k2_shared_experts"]
        assert c.num_experts_per_tok == p["k2_experts_per_token"]
        assert [c.n_routed_experts, c.hidden] == p["k2_router_weight_shape"]
        assert c.routed_scaling_factor == p["k2_routed_scaling_factor"]
        assert c.norm_topk_prob == p["k2_norm_topk_prob"]
    assert W.CONFIGS["k2_decode_bf16"].n_group == p["k2_n_group"]
    assert W.CONFIGS["k2_decode_bf16"].topk_group == p["k2_topk_group"]
    v4 = W.CONFIGS["v4_fp4"]
    assert (v4.hidden, v4.n_routed_experts, v4.num_experts_per_tok) == (
        p["v4_hidden"], p["v4_routed_experts"], p["v4_experts_per_token"])
    assert v4.routed_scaling_factor == p["v4_route_scale"] and v4.score_fn == p["v4_score"]
    mx = W.CONFIGS["mx896"]
    assert (mx.n_routed_experts, mx.num_experts_per_tok, mx.n_shared_experts) == (
        p["mx_routed_experts"], p["mx_experts_per_token"], p["mx_shared_experts"])


def test_mx_storage_arithmetic():
    """4 bits per element plus one 8-bit scale per 32 elements = 17/32 byte per
    parameter; the pages' 2.78T parameters then need 1.477 TB, between their
    4-bit floor (1.39 TB) and the repository size (1.56 TB)."""
    p = page()
    c = W.CONFIGS["mx896"]
    P = 3 * c.hidden * c.moe_intermediate_size
    assert W.weight_bytes_per_matrix(c, c.moe_intermediate_size) * 32 == P * 17
    floor = p["mx_total_params"] * 4 / 8
    assert abs(floor - p["mx_4bit_floor_bytes"]) / p["mx_4bit_floor_bytes"] < 0.01
    mx = p["mx_total_params"] * 17 / 32
    assert p["mx_4bit_floor_bytes"] < mx < p["mx_repo_bytes"]
    assert p["mx_total_params"] * 2 >= p["mx_16bit_bytes_at_least"]


@pytest.mark.parametrize("wfmt", ["fp8_e4m3_b128x128", "fp4_e2m1_ue8m0_b32", "mxfp4"])
def test_weight_encoder_writes_valid_codes(wfmt):
    g = torch.Generator().manual_seed(0)
    w = torch.randn(1, 128, 256, generator=g) * 0.02
    data, scale = W.encode_weight(w, wfmt)
    d, s = data.numpy(), scale.numpy()
    ref = w[0].double().numpy()
    rows = [0, 5, 64, 127]
    dec = np.array([[oracle.weight_value(wfmt, d, s, 128, 256, 0, r, c) for c in range(256)]
                    for r in rows])
    if wfmt == "fp8_e4m3_b128x128":
        assert np.all(np.abs(dec - ref[rows]) <= np.abs(ref[rows]) * 2 ** -4 + 1e-9)
    else:
        # every block's scale follows its rule, and each value is within one grid step
        for i, r in enumerate(rows):
            for b in range(8):
                amax = np.abs(ref[r, b * 32:(b + 1) * 32]).max()
                e = int(s[0, r, b]) - 127
                if wfmt == "fp4_e2m1_ue8m0_b32":
                    assert e == oracle.pow2_ceil_exp(amax, 6.0)
                else:
                    assert e == oracle.floor_log2(amax) - 2
                err = np.abs(dec[i, b * 32:(b + 1) * 32] - ref[r, b * 32:(b + 1) * 32])
                # half the top grid step (4 -> 6) is one scale unit; the OCP MX rule
                # leaves amax/X in [4, 8), so values above 6X saturate (error < 2X)
                bound = 1.0 if wfmt == "fp4_e2m1_ue8m0_b32" else 2.0
                assert np.all(err <= 2.0 ** e * bound + 1e-12)


def test_inputs_are_seeded_and_shaped():
    c = W.CONFIGS["tiny_bf16"]
    a, b = W.make_inputs(c), W.make_inputs(c)
    assert torch.equal(a["x"].view(torch.int16), b["x"].view(torch.int16))
    assert a["x"].shape == (c.T, c.hidden) and a["x"].dtype == torch.bfloat16
    assert a["gate_w"].shape == (c.n_routed_experts, c.hidden)
    assert a["gate_bias"].abs().max() <= W.BIAS_UNIFORM_HALF_WIDTH
    wts = W.make_weights(c)
    assert wts["w13"].shape == (16, 256, 256) and wts["w2"].shape == (16, 256, 128)
    assert wts["sh_w13"].shape == (1, 256, 256)
    part = W.make_weights(c, experts=[3])
    assert torch.equal(part["w13"][3].view(torch.int16), wts["w13"][3].view(torch.int16))
    assert torch.count_nonzero(part["w13"][2].float()) == 0


def test_balanced_recipe_reduced_size():
    """The balanced recipe on a reduced shape (same 8/4 grouping): loads are
    within 20% of the mean, measured with the oracle's routing."""
    c = W.CONFIGS["k2_prefill_fp8w"].replace(T=2048, hidden=512, n_routed_experts=64)
    inp = W.make_inputs(c)
    r = oracle.route(c, W.bf16_codes(inp["x"]), inp["gate_w"].numpy(), inp["gate_bias"].numpy())
    counts = np.bincount(r["idx"].ravel(), minlength=c.n_routed_experts)
    m = counts.mean()
    assert counts.max() <= 1.2 * m and counts.min() >= 0.8 * m
