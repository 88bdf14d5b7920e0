"""GPU parity of the prologue (post-attention RMSNorm fused with the expert-input
quantisation, "DeepSeek V3架构拆解…" 三 decoder layer; "DeepSeek-V4-Pro 架构与代码
概述" 文件说明 model.py RMSNorm / kernel.py act_quant_kernel) and of the layer
run from the un-normalised hidden state, against the float64 oracle, through
the C ABI.

Both sides round the normalised value to bf16 from double precision; they may
differ only where the oracle reports a rounding near-tie (within 2^-36 of a
bf16 midpoint). Such elements are left out of the exact comparison and their
tokens out of the exact routing and output comparisons."""
import numpy as np
import pytest
import torch

import expert_routing_grouped_layer_b200 as moe
import oracle
from expert_routing_grouped_layer_b200 import workloads as W
from moe_testlib import LAYER_TOL, compare_routing, rel_l2_rows

pytestmark = pytest.mark.gpu


def _prologue(cfg, x, w, eps):
    T, H = x.shape
    xn = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    q = qs = None
    if cfg.afmt != "bf16":
        q = torch.empty(T, H, dtype=torch.uint8, device="cuda")
        qs = torch.empty(T, H // 32, dtype=torch.uint8, device="cuda")
    moe.moe_rmsnorm_prologue(cfg, x, T, w, eps, xn, q, qs)
    torch.cuda.synchronize()
    return xn, q, qs


def _check_prologue(cfg, x, w, eps):
    xn, q, qs = _prologue(cfg, x, w, eps)
    want, near = oracle.rmsnorm(W.bf16_codes(x), w.cpu().numpy(), eps)
    got = W.bf16_codes(xn)
    ok = ~near
    assert np.array_equal(got[ok], want[ok])
    if cfg.afmt != "bf16":
        clean = ~near.any(axis=1)  # tokens whose every normalised value is fixed
        _, q_ref, s_ref = oracle.expert_input(cfg.afmt, want[clean])
        blk = 128 if cfg.afmt == "fp8_e4m3_pow2_b128" else 32
        assert np.array_equal(q.cpu().numpy()[clean], q_ref)
        assert np.array_equal(qs.cpu().numpy()[clean], np.repeat(s_ref, blk // 32, axis=1))
    return int(near.sum())


@pytest.mark.parametrize("afmt", ["bf16", "fp8_e4m3_pow2_b128", "mxfp8"])
def test_prologue_bit_exact_with_edge_rows(afmt):
    cfg = W.CONFIGS["tiny_bf16"].replace(hidden=1024, afmt=afmt,
                                         wfmt="bf16" if afmt == "bf16" else "mxfp4")
    T, H = 300, cfg.hidden
    g = torch.Generator(device="cuda").manual_seed(21)
    xf = torch.randn(T, H, generator=g, device="cuda") * torch.exp2(
        torch.randint(-30, 30, (T, 1), generator=g, device="cuda").float())
    xf[0] = 0.0  # zero row: r = 1/sqrt(eps), every output 0
    xf[1] = 3.0  # constant row
    xf[2, :] = 0.0
    xf[2, 17] = -2.5e38  # one element near the top of the bf16 range
    xf[3] = xf[3] * 1e-30  # tiny magnitudes
    x = xf.to(torch.bfloat16)
    w = (1.0 + 0.3 * torch.randn(H, generator=g, device="cuda")).float()
    w[5] = 0.0
    w[6] = -1.5
    _check_prologue(cfg, x, w, 1e-6)
    _check_prologue(cfg, x, w, 0.5)  # eps large enough to matter on most rows


def test_prologue_full_size_896_experts():
    """The 896-expert layer's 16384 x 7168 hidden state, MXFP8 codes included."""
    cfg = W.CONFIGS["mx896"]
    inp = W.make_inputs(cfg, "cuda")
    x, w, eps = W.make_prenorm_inputs(cfg, inp["x"])
    _check_prologue(cfg, x, w, eps)


_LAYER_CASES = {
    "bf16": W.CONFIGS["tiny_bf16"],
    "fp8w": W.CONFIGS["tiny_bf16"].replace(T=300, hidden=512, moe_intermediate_size=256,
                                           shared_intermediate_size=256, n_routed_experts=8,
                                           num_experts_per_tok=3, wfmt="fp8_e4m3_b128x128"),
    "fp4": W.CONFIGS["tiny_bf16"].replace(T=300, hidden=1024, moe_intermediate_size=512,
                                          shared_intermediate_size=512, n_routed_experts=8,
                                          num_experts_per_tok=3, wfmt="fp4_e2m1_ue8m0_b32",
                                          afmt="fp8_e4m3_pow2_b128", score_fn="sqrtsoftplus",
                                          routed_scaling_factor=2.5),
    "mx": W.CONFIGS["tiny_bf16"].replace(T=300, hidden=1024, moe_intermediate_size=512,
                                         shared_intermediate_size=512, n_routed_experts=8,
                                         num_experts_per_tok=3, wfmt="mxfp4", afmt="mxfp8",
                                         n_shared_experts=2),
    "decode_full": W.CONFIGS["k2_decode_bf16"],
}


@pytest.mark.parametrize("name", list(_LAYER_CASES))
def test_layer_from_the_unnormalised_state(name):
    """moe_layer_forward_prenorm against the oracle run on its own RMSNorm output
    (routing of every token, every token's output), and bit for bit against
    moe_layer_forward on the prologue's x_norm."""
    cfg = _LAYER_CASES[name]
    inp = W.make_inputs(cfg, "cuda")
    wts = W.make_weights(cfg, "cuda")
    x, nw, eps = W.make_prenorm_inputs(cfg, inp["x"])
    T, k, E = cfg.T, cfg.num_experts_per_tok, cfg.n_routed_experts
    layer = moe.MoELayer(cfg, wts, inp["gate_w"], inp["gate_bias"], max_tokens=T, device="cuda")
    out = layer.forward_prenorm(x, nw, eps).clone()
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    xn_gpu = layer.intermediate(T, moe.WS_X_NORM, torch.bfloat16, (T, cfg.hidden)).clone()
    idx = layer.intermediate(T, moe.WS_TOPK_IDX, torch.int32, (T, k)).cpu().numpy()
    tw = layer.intermediate(T, moe.WS_TOPK_W, torch.float32, (T, k)).cpu().numpy()
    # the same layer on the prologue's output, through the plain entry point
    out2 = layer.forward(xn_gpu).clone()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    # the oracle: its own RMSNorm, routing and layer
    xn, near = oracle.rmsnorm(W.bf16_codes(x), nw.cpu().numpy(), eps)
    assert np.array_equal(W.bf16_codes(xn_gpu)[~near], xn[~near])
    clean = ~near.any(axis=1)
    r = oracle.route(cfg, xn, inp["gate_w"].cpu().numpy(), inp["gate_bias"].cpu().numpy())
    toks = np.nonzero(clean)[0]
    compare_routing(cfg, {"idx": idx, "w": tw}, {k_: v[toks] for k_, v in r.items()}, toks)
    ok = toks[~r["near_tie"][toks]]
    want = oracle.layer(cfg, xn[ok], r["idx"][ok], r["w"][ok], lambda e: W.expert_slice(wts, e),
                        lambda s: W.expert_slice(wts, s, shared=True))
    err = rel_l2_rows(out.float().cpu().numpy().astype(np.float64)[ok], want)
    assert err.max() <= LAYER_TOL[cfg.afmt], (float(err.max()), int(ok[err.argmax()]))
