"""GPU parity of the quantised-weight / quantised-activation layers against the
float64 oracle (which decodes the same stored bytes), through the C ABI."""
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


def _layer_check(cfg, T=None, sample=None, seed=0):
    """Routing of every token against the oracle (sets and weights, near-ties
    excepted), the permutation element by element, and the layer output token
    by token: every token when sample is None, else the chosen tokens (a seeded
    sample plus the tokens at ragged tile ends)."""
    T = cfg.T if T is None else T
    inp = W.make_inputs(cfg, "cuda")
    wts = W.make_weights(cfg, "cuda")
    g = gpu_forward(cfg, inp, wts, T)
    assert g["status"] == 0
    r = oracle_route(cfg, inp, T=T)  # every token
    compare_routing(cfg, g, r, np.arange(T))
    check_permutation_properties(cfg, g, T)
    compare_permutation_exact(cfg, g, r)
    if sample is None:
        toks = np.nonzero(~r["near_tie"])[0]
    else:
        toks = chosen_tokens(cfg, g, r, sample, seed)
    err = check_layer_tokens(cfg, inp, wts, g, r, toks, LAYER_TOL[cfg.afmt])
    return g, float(err.max())


FP8_TINY = W.CONFIGS["tiny_bf16"].replace(wfmt="fp8_e4m3_b128x128")


def test_fp8_weights_tiny():
    _layer_check(FP8_TINY)


@pytest.mark.parametrize("T", [1, 29])
def test_fp8_weights_tiny_ragged(T):
    _layer_check(FP8_TINY, T=T)


def test_fp8_weights_several_tiles():
    cfg = FP8_TINY.replace(T=700, hidden=512, moe_intermediate_size=256,
                           shared_intermediate_size=256, n_routed_experts=8,
                           num_experts_per_tok=3, n_shared_experts=2)
    _layer_check(cfg)


def test_fp8_weights_group_limited_prefill_full_size():
    cfg = W.CONFIGS["k2_prefill_fp8w"]
    g, err = _layer_check(cfg, sample=8, seed=1)
    counts = np.diff(g["offsets"])
    m = counts.mean()
    # the workload's balanced recipe: every expert within 20% of the mean load
    assert counts.min() >= 0.8 * m and counts.max() <= 1.2 * m


# ----------------------------------------------------------- activation quantisers
def _x_with_edge_cases(T, H, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn(T, H, generator=g, device="cuda") * torch.exp2(
        torch.randint(-20, 20, (T, 1), generator=g, device="cuda").float())
    x[0, :128] = 0.0  # an all-zero block
    x[1, :32] = 448.0 * 2.0 ** 3  # exact power-of-two edge
    x[2, 5] = 3.0e38  # near the top of the bf16 range
    x[3, :64] = 1.0e-39  # subnormal block
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("afmt,blk", [("fp8_e4m3_pow2_b128", 128), ("mxfp8", 32)])
def test_quantize_activations_bit_exact(afmt, blk):
    cfg = W.CONFIGS["tiny_bf16"].replace(hidden=1024, afmt=afmt, wfmt="mxfp4")
    T, H = 40, cfg.hidden
    x = _x_with_edge_cases(T, H, 3)
    xq = torch.empty(T, H, dtype=torch.uint8, device="cuda")
    xs = torch.empty(T, H // blk, dtype=torch.uint8, device="cuda")
    moe.moe_quantize_activations(cfg, x, T, xq, xs)
    torch.cuda.synchronize()
    _, q_ref, s_ref = oracle.expert_input(afmt, W.bf16_codes(x))
    assert np.array_equal(xs.cpu().numpy(), s_ref)
    assert np.array_equal(xq.cpu().numpy(), q_ref)


@pytest.mark.parametrize("afmt,blk", [("fp8_e4m3_pow2_b128", 128), ("mxfp8", 32)])
def test_pack_expert_inputs_gathers_and_repeats_scales(afmt, blk):
    cfg = W.CONFIGS["tiny_bf16"].replace(hidden=1024, afmt=afmt, wfmt="mxfp4")
    T, k, H = 24, cfg.num_experts_per_tok, cfg.hidden
    N = T * k
    x = _x_with_edge_cases(T, H, 4)
    g = torch.Generator(device="cuda").manual_seed(5)
    sp = torch.randperm(N, generator=g, device="cuda").to(torch.int32)
    xa = torch.empty(N + T, H, dtype=torch.uint8, device="cuda")
    xs = torch.empty(N + T, H // 32, dtype=torch.uint8, device="cuda")
    moe.moe_pack_expert_inputs(cfg, x, T, sp, xa, xs)
    torch.cuda.synchronize()
    _, q_ref, s_ref = oracle.expert_input(afmt, W.bf16_codes(x))
    tok = np.concatenate([sp.cpu().numpy() // k, np.arange(T)])
    assert np.array_equal(xa.cpu().numpy(), q_ref[tok])
    assert np.array_equal(xs.cpu().numpy(), np.repeat(s_ref[tok], blk // 32, axis=1))


# ----------------------------------------------------------- block-scaled layers
FP4_TINY = W.CONFIGS["tiny_bf16"].replace(
    hidden=512, moe_intermediate_size=512, shared_intermediate_size=512,
    wfmt="fp4_e2m1_ue8m0_b32", afmt="fp8_e4m3_pow2_b128", score_fn="sqrtsoftplus",
    routed_scaling_factor=2.5)
MX_TINY = W.CONFIGS["tiny_bf16"].replace(
    hidden=512, moe_intermediate_size=512, shared_intermediate_size=512, wfmt="mxfp4",
    afmt="mxfp8", n_shared_experts=2)


@pytest.mark.parametrize("cfg", [FP4_TINY, MX_TINY], ids=["fp4_pow2", "mx"])
def test_block_scaled_tiny(cfg):
    _layer_check(cfg)


@pytest.mark.parametrize("cfg", [FP4_TINY, MX_TINY], ids=["fp4_pow2", "mx"])
def test_block_scaled_several_tiles_ragged(cfg):
    # ~260 rows per expert: several 64- and 128-token tiles with ragged ends,
    # H = 1024 -> 8 down-projection tiles and 8 K stages of the gate/up GEMM
    _layer_check(cfg.replace(T=700, hidden=1024, n_routed_experts=8, num_experts_per_tok=3))


@pytest.mark.parametrize("T", [1, 13])
def test_block_scaled_few_tokens(T):
    _layer_check(MX_TINY, T=T)


def test_v4_fp4_full_size():
    cfg = W.CONFIGS["v4_fp4"]
    _layer_check(cfg, sample=8, seed=2)


def test_mx896_full_size_zipf():
    cfg = W.CONFIGS["mx896"]
    g, _ = _layer_check(cfg, sample=6, seed=3)
    counts = np.diff(g["offsets"])
    assert counts.max() > 10 * counts.mean()  # hot experts take >10x the mean


def test_fp8_weights_extreme_row_magnitudes():
    """FP8 weights run gate/up on f16 operands, each token row scaled by its own
    power of two: rows from 2^-30 to 2^30 times the usual magnitude (far outside
    f16's range unscaled) and a row whose elements span 2^30 must still match the
    oracle row by row. Routing comes from the unscaled inputs and is passed to
    both sides, so only the expert computation sees the extreme rows."""
    cfg = FP8_TINY.replace(T=96, hidden=512, moe_intermediate_size=256,
                           shared_intermediate_size=256, n_routed_experts=8,
                           num_experts_per_tok=3, n_shared_experts=2)
    T, H, k = cfg.T, cfg.hidden, cfg.num_experts_per_tok
    dev = torch.device("cuda")
    inp = W.make_inputs(cfg, dev)
    wts = W.make_weights(cfg, dev)
    r = oracle_route(cfg, inp, T=T)
    g = torch.Generator(device="cpu").manual_seed(11)
    row_exp = torch.tensor([-30, -17, -8, 0, 9, 16, 30], dtype=torch.float64)[
        torch.randint(0, 7, (T,), generator=g)]
    xs = inp["x"].double().cpu() * torch.exp2(row_exp)[:, None]
    xs[5] = inp["x"][5].double().cpu() * torch.exp2(
        torch.randint(-20, 11, (H,), generator=g).double())  # one row spanning 2^30
    x_big = xs.to(torch.bfloat16).to(dev)
    layer = moe.MoELayer(cfg, wts, inp["gate_w"], inp["gate_bias"], max_tokens=T, device=dev)
    P = lambda which: layer.ws_ptr(T, which)
    st, ws, ccfg, cw = layer.status, layer.ws, layer.ccfg, layer.cw
    idx = torch.as_tensor(r["idx"], dtype=torch.int32, device=dev).contiguous()
    w = torch.as_tensor(r["w"], dtype=torch.float32, device=dev).contiguous()
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    moe.moe_permute(ccfg, idx, T, P(moe.WS_OFFSETS), P(moe.WS_SORTED_PAIR), P(moe.WS_ROW_OF), st,
                    ws, ws.numel())
    moe.moe_pack_expert_inputs(ccfg, x_big, T, P(moe.WS_SORTED_PAIR), P(moe.WS_XA),
                               P(moe.WS_XA_SCALE))
    moe.moe_expert_gate_up(ccfg, P(moe.WS_XA), P(moe.WS_XA_SCALE), T, P(moe.WS_OFFSETS), cw,
                           P(moe.WS_H), P(moe.WS_H_SCALE), st)
    moe.moe_expert_down(ccfg, P(moe.WS_H), P(moe.WS_H_SCALE), T, P(moe.WS_OFFSETS), cw,
                        P(moe.WS_Y), P(moe.WS_SHARED_Y), st)
    moe.moe_combine(ccfg, P(moe.WS_Y), P(moe.WS_SHARED_Y), P(moe.WS_ROW_OF), w, T, out)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    want = oracle.layer(cfg, W.bf16_codes(x_big), r["idx"], r["w"],
                        lambda e: W.expert_slice(wts, e), lambda s: W.expert_slice(wts, s, shared=True))
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.linalg.norm(got - want, axis=1) / np.maximum(np.linalg.norm(want, axis=1), 1e-300)
    assert err.max() <= LAYER_TOL["bf16"], (err.max(), int(err.argmax()))


def test_fp8_weights_h_rows_are_f16_with_row_exponents():
    """With FP8 weights the gate/up call leaves h as f16 rows holding the bf16
    SwiGLU output times 2^-e, e per row in h_scale: the row's largest magnitude
    lands in [2^13, 2^14), every element within 2^-30 of it converts back to a
    bf16 value exactly, and the rows match the oracle's SwiGLU output (its
    expert computation with an identity down projection, E4M3 1.0 on the
    diagonal with unit block scales) to bf16 rounding plus fp32 summation."""
    cfg = FP8_TINY.replace(T=80, hidden=512, moe_intermediate_size=256, shared_intermediate_size=256,
                           n_routed_experts=8, num_experts_per_tok=3, n_shared_experts=1)
    T, H, I, k, S = cfg.T, cfg.hidden, cfg.moe_intermediate_size, cfg.num_experts_per_tok, 1
    N = T * k
    dev = torch.device("cuda")
    inp = W.make_inputs(cfg, dev)
    wts = W.make_weights(cfg, dev)
    r = oracle_route(cfg, inp, T=T)
    layer = moe.MoELayer(cfg, wts, inp["gate_w"], inp["gate_bias"], max_tokens=T, device=dev)
    P = lambda which: layer.ws_ptr(T, which)
    st, ws, ccfg, cw = layer.status, layer.ws, layer.ccfg, layer.cw
    idx = torch.as_tensor(r["idx"], dtype=torch.int32, device=dev).contiguous()
    moe.moe_permute(ccfg, idx, T, P(moe.WS_OFFSETS), P(moe.WS_SORTED_PAIR), P(moe.WS_ROW_OF), st,
                    ws, ws.numel())
    moe.moe_pack_expert_inputs(ccfg, inp["x"], T, P(moe.WS_SORTED_PAIR), P(moe.WS_XA),
                               P(moe.WS_XA_SCALE))
    moe.moe_expert_gate_up(ccfg, P(moe.WS_XA), P(moe.WS_XA_SCALE), T, P(moe.WS_OFFSETS), cw,
                           P(moe.WS_H), P(moe.WS_H_SCALE), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    view = lambda which, n, dt: ws[P(which) - ws.data_ptr():][: n * torch.tensor([], dtype=dt).element_size()].view(dt)
    h = view(moe.WS_H, (N + S * T) * I, torch.float16).view(N + S * T, I).double().cpu().numpy()
    e = view(moe.WS_H_SCALE, N + S * T, torch.int8).cpu().numpy().astype(np.int64)
    sp = view(moe.WS_SORTED_PAIR, N, torch.int32).cpu().numpy()
    rec = h * np.exp2(e)[:, None]
    # the oracle's SwiGLU rows: identity down projection in the weights' own format
    w2_id = np.zeros((1, H, I), np.uint8)
    w2_id[0, np.arange(I), np.arange(I)] = oracle.e4m3_encode(np.ones(1))[0]
    w2s_id = np.ones((1, H // 128, I // 128), np.float32)
    xin, _, _ = oracle.expert_input(cfg.afmt, W.bf16_codes(inp["x"]))
    want = np.zeros_like(rec)
    for row in range(N + S * T):
        t, ex = (sp[row] // k, int(r["idx"][sp[row] // k][sp[row] % k])) if row < N else (row - N, None)
        w13, w13s, _, _ = W.expert_slice(wts, ex) if ex is not None else W.expert_slice(wts, 0, shared=True)
        want[row] = oracle.expert_rows(cfg.wfmt, cfg.afmt, w13, w13s, w2_id, w2s_id, 0, I, H,
                                       xin[t:t + 1])[0, :I]
    for row in range(N + S * T):
        m = np.abs(rec[row]).max()
        if m == 0:
            assert e[row] == 0
            continue
        if e[row] > -127:
            assert 2.0 ** 13 <= np.abs(h[row]).max() < 2.0 ** 14, row
        big = np.abs(rec[row]) >= m * 2.0 ** -30
        as_bf16 = torch.tensor(rec[row][big]).to(torch.bfloat16).double().numpy()
        assert np.array_equal(as_bf16, rec[row][big]), row
    err = np.linalg.norm(rec - want, axis=1) / np.maximum(np.linalg.norm(want, axis=1), 1e-300)
    assert err.max() <= 2.0 ** -7, (err.max(), int(err.argmax()))


@pytest.mark.parametrize("name", ["bf16", "fp8w", "fp4", "mx"])
def test_swiglu_limit_every_format(name):
    """swiglu_limit = 0.25, below the typical |g| and |u| of these inputs, so the
    clamp changes many features: the layer still matches the oracle."""
    base = {"bf16": W.CONFIGS["tiny_bf16"], "fp8w": FP8_TINY, "fp4": FP4_TINY, "mx": MX_TINY}[name]
    _layer_check(base.replace(swiglu_limit=0.25))
