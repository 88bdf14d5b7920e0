"""GPU parity of the NVFP4 layer ("DeepSeek V3架构拆解…", 四 NVFP4 量化: routed
experts' weights and input activations in E2M1 with an E4M3 scale per 16
elements and a per-tensor fp32 scale; the shared experts stay bf16) against the
float64 oracle, which decodes the same stored bytes, through the C ABI."""
import numpy as np
import pytest
import torch

import expert_routing_grouped_layer_b200 as moe
import oracle
from expert_routing_grouped_layer_b200 import workloads as W
from moe_testlib import (LAYER_TOL, check_layer_tokens, check_permutation_properties,
                         chosen_tokens, compare_permutation_exact, compare_routing, gpu_forward,
                         oracle_route)

pytestmark = pytest.mark.gpu

NV_TINY = W.CONFIGS["tiny_bf16"].replace(hidden=512, moe_intermediate_size=256,
                                         shared_intermediate_size=256, wfmt="nvfp4",
                                         afmt="nvfp4")


def _check(cfg, T=None, sample=None, seed=0):
    T = cfg.T if T is None else T
    inp = W.make_inputs(cfg, "cuda")
    wts = W.make_weights(cfg, "cuda")
    g = gpu_forward(cfg, inp, wts, T)
    assert g["status"] == 0
    r = oracle_route(cfg, inp, T=T)
    compare_routing(cfg, g, r, np.arange(T))
    check_permutation_properties(cfg, g, T)
    compare_permutation_exact(cfg, g, r)
    toks = np.nonzero(~r["near_tie"])[0] if sample is None else chosen_tokens(cfg, g, r, sample, seed)
    err = check_layer_tokens(cfg, inp, wts, g, r, toks, LAYER_TOL["nvfp4"])
    return g, float(err.max())


def _pack_codes(q):
    """One E2M1 code per byte -> two per byte, even element in the low nibble."""
    return (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)


def test_nvfp4_activation_quantiser_bit_exact():
    cfg = NV_TINY.replace(hidden=1024)
    T, H = 48, cfg.hidden
    g = torch.Generator(device="cuda").manual_seed(9)
    xf = torch.randn(T, H, generator=g, device="cuda") * torch.exp2(
        torch.randint(-12, 6, (T, 1), generator=g, device="cuda").float())
    xf[0, :16] = 0.0  # a zero group
    xf[1, :16] = -0.0
    xf[2, 3] = 1.0e4  # a group whose scale saturates at 448
    xf[3, :32] = 1.0e-30  # groups whose scale underflows to zero
    xf[4, 16:32] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 2)  # grid midpoints
    x = xf.to(torch.bfloat16)
    xq = torch.empty(T, H // 2, dtype=torch.uint8, device="cuda")
    xs = torch.empty(T, H // 16, dtype=torch.uint8, device="cuda")
    moe.moe_quantize_activations(cfg, x, T, xq, xs)
    torch.cuda.synchronize()
    gx, _ = W.nvfp4_act_scales()
    vals = oracle.bf16_value_rows(W.bf16_codes(x))
    for t in range(T):
        q, sc = oracle.quant_nvfp4(vals[t], gx)
        assert np.array_equal(xs[t].cpu().numpy(), sc), t
        assert np.array_equal(xq[t].cpu().numpy(), _pack_codes(q)), t


def test_nvfp4_tiny_layer():
    _check(NV_TINY)


@pytest.mark.parametrize("T", [1, 13])
def test_nvfp4_few_tokens(T):
    _check(NV_TINY, T=T)


@pytest.mark.parametrize("S", [0, 2])
def test_nvfp4_several_tiles_ragged(S):
    # ~260 rows per expert: three 96-token tiles with a ragged end; H = 1024 ->
    # four 256-row down-projection units and four K stages of the gate/up GEMM
    _check(NV_TINY.replace(T=700, hidden=1024, moe_intermediate_size=512,
                           shared_intermediate_size=512, n_routed_experts=8,
                           num_experts_per_tok=3, n_shared_experts=S))


def test_nvfp4_full_size():
    cfg = W.CONFIGS["k2_nvfp4"]
    _check(cfg, sample=8, seed=5)


def test_nvfp4_token_order_permutes_output_bit_for_bit():
    cfg = NV_TINY.replace(T=300, hidden=1024, moe_intermediate_size=512,
                          shared_intermediate_size=512, n_routed_experts=8, num_experts_per_tok=3)
    inp = W.make_inputs(cfg, "cuda")
    wts = W.make_weights(cfg, "cuda")
    layer = moe.MoELayer(cfg, wts, inp["gate_w"], inp["gate_bias"], max_tokens=cfg.T, device="cuda")
    out = layer.forward(inp["x"]).clone()
    perm = torch.randperm(cfg.T, generator=torch.Generator().manual_seed(3)).to("cuda")
    out_p = layer.forward(inp["x"][perm].contiguous()).clone()
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    assert torch.equal(out_p.view(torch.int16), out[perm].view(torch.int16))
