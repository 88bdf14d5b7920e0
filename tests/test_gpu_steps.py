"""GPU parity of single steps against the oracle, on synthetic step inputs with
no routing in the loop: the dispatch permutation on both sides of its
one-chunk path, the weighted combine on both sides of its small-batch path,
and the f16 expert-input rows that FP8-weight layers feed to the f16
tensor-core gate/up GEMM. Also the pipeline waits' time limit: a wait that
nothing ends reports a timeout and leaves the context usable."""
import time

import numpy as np
import pytest
import torch

import expert_routing_grouped_layer_b200 as moe
import oracle
from expert_routing_grouped_layer_b200 import workloads as W

pytestmark = pytest.mark.gpu

TINY = W.CONFIGS["tiny_bf16"]
PERM_CHUNK = 4096  # pairs handled by one permutation CTA


# (T, k, E): N = T*k at 1, exactly one chunk, one pair past it, and many chunks
@pytest.mark.parametrize("T,k,E", [(1, 1, 16), (512, 8, 384), (1024, 4, 16), (1025, 4, 16),
                                   (2049, 2, 1024), (7000, 6, 384)])
def test_permute_exact_around_one_chunk(T, k, E):
    cfg = TINY.replace(T=T, n_routed_experts=E, num_experts_per_tok=k, n_group=1, topk_group=1)
    g = torch.Generator().manual_seed(T * 7 + E)
    idx = torch.randint(0, E, (T, k), generator=g, dtype=torch.int32)
    hot = torch.rand(T, k, generator=g) < 0.5  # half the pairs on three experts
    idx[hot] = torch.randint(0, min(E, 3), (int(hot.sum()),), generator=g, dtype=torch.int32)
    dev = torch.device("cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sp = torch.empty(T * k, dtype=torch.int32, device=dev)
    ro = torch.empty(T * k, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(moe.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device=dev)
    moe.moe_permute(cfg, idx.to(dev), T, off, sp, ro, st, ws, ws.numel())
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    w_off, w_sp, w_ro = oracle.permute(idx.numpy(), E)
    assert np.array_equal(off.cpu().numpy(), w_off)
    assert np.array_equal(sp.cpu().numpy(), w_sp)
    assert np.array_equal(ro.cpu().numpy(), w_ro)


def _bf16(t):
    return t.to(torch.bfloat16)


def test_combine_around_small_batch_path():
    """The combine switches kernels at 8 CTAs per SM worth of tokens; both sides,
    a ragged second 128-column block (H/8 = 144), skipped pairs (row_of = -1)
    and two shared experts, against the oracle's float64 sum. The GPU sums in
    fp32 and rounds once to bf16: each element is within 2^-8 of the result plus
    2^-20 of the sum of the terms' magnitudes (fp32 summation, where terms cancel)."""
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    thr = 8 * n_sms
    H, k, S = 1152, 6, 2
    cfg = TINY.replace(hidden=H, num_experts_per_tok=k, n_shared_experts=S)
    dev = torch.device("cuda")
    for T in (1, thr - 1, thr, thr + 517):
        g = torch.Generator().manual_seed(T)
        N = T * k
        y = _bf16(torch.randn(N, H, generator=g) * torch.exp2(torch.randint(-6, 6, (N, 1), generator=g)))
        ys = _bf16(torch.randn(S, T, H, generator=g))
        ro = torch.randperm(N, generator=g).to(torch.int32)
        ro[torch.rand(N, generator=g) < 0.05] = -1
        w = torch.rand(T, k, generator=g, dtype=torch.float32)
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        moe.moe_combine(cfg, y.to(dev), ys.to(dev), ro.to(dev), w.to(dev), T, out)
        torch.cuda.synchronize()
        rows = ro.long().clamp(min=0)
        yg = y.double()[rows].view(T, k, H) * (ro >= 0).double().view(T, k, 1)
        want = oracle.combine(w.double().numpy(), yg.numpy(), ys.double().numpy())
        mag = oracle.combine(w.double().abs().numpy(), yg.abs().numpy(), ys.double().abs().numpy())
        got = out.double().cpu().numpy()
        bad = np.abs(got - want) > 2.0 ** -8 * np.abs(want) + 2.0 ** -20 * mag
        assert not bad.any(), (T, int(bad.sum()))


def test_pack_f16_rows_are_exact():
    """FP8-weight layers get f16 rows x * 2^-e with e per row: reconstructing
    xa * 2^e gives the bf16 rows back bit for bit for every element within
    2^-30 of its row's largest, the largest lands in [2^13, 2^14) unless e is
    clamped at -127, and an all-zero row has e = 0."""
    cfg = TINY.replace(hidden=512, n_routed_experts=8, num_experts_per_tok=3,
                       wfmt="fp8_e4m3_b128x128", n_shared_experts=1)
    T, k, H = 40, cfg.num_experts_per_tok, cfg.hidden
    N = T * k
    g = torch.Generator().manual_seed(9)
    x = torch.randn(T, H, generator=g) * torch.exp2(torch.randint(-40, 40, (T, 1), generator=g).float())
    x[0] = 0.0                                        # all-zero row
    x[1] = torch.randn(H, generator=g) * 1e-39         # bf16 subnormals: e clamps at -127
    x[2, :] = 0.0
    x[2, 7] = 3.0e38                                   # near the top of the bf16 range
    x[2, 8] = 1.0                                      # far below it: rounds in f16
    x[3] = torch.randn(H, generator=g) * torch.exp2(torch.randint(-28, 2, (H,), generator=g).float())
    dev = torch.device("cuda")
    xb = _bf16(x).to(dev)
    sp = torch.randperm(N, generator=g).to(torch.int32).to(dev)
    xa = torch.empty(N + T, H, dtype=torch.float16, device=dev)
    xs = torch.empty(N + T, dtype=torch.int8, device=dev)
    moe.moe_pack_expert_inputs(cfg, xb, T, sp, xa, xs)
    torch.cuda.synchronize()
    tok = np.concatenate([sp.cpu().numpy() // k, np.arange(T)])
    e = xs.cpu().numpy().astype(np.int64)
    rec = xa.double().cpu().numpy() * np.exp2(e)[:, None]
    want = xb.double().cpu().numpy()[tok]
    rmax = np.abs(want).max(axis=1)
    for r in range(N + T):
        if rmax[r] == 0:
            assert e[r] == 0 and not rec[r].any()
            continue
        if e[r] > -127:
            assert 2.0 ** 13 <= rmax[r] * 2.0 ** -e[r] < 2.0 ** 14
        big = np.abs(want[r]) >= rmax[r] * 2.0 ** -30
        assert np.array_equal(rec[r][big], want[r][big]), r
        assert np.all(np.abs(rec[r] - want[r]) <= 2.0 ** (e[r] - 25)), r


def test_wait_limit_reports_timeout_and_context_stays_usable():
    """A bounded pipeline wait on a barrier nothing arrives on gives up after its
    limit (2 s) and reports MOE_DEV_TIMEOUT in the status word, without a trap;
    the same context then runs a layer that still matches the oracle."""
    dev = torch.device("cuda")
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moe.moe_selftest_wait_limit(st)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert int(st.item()) & moe.MOE_DEV_TIMEOUT
    assert 1.5 < waited < 60.0, waited
    cfg = TINY
    inp = W.make_inputs(cfg, dev)
    wts = W.make_weights(cfg, dev)
    layer = moe.MoELayer(cfg, wts, inp["gate_w"], inp["gate_bias"], max_tokens=cfg.T, device=dev)
    out = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    r = oracle.route(cfg, W.bf16_codes(inp["x"]), inp["gate_w"].cpu().numpy(),
                     inp["gate_bias"].cpu().numpy())
    want = oracle.layer(cfg, W.bf16_codes(inp["x"]), r["idx"], r["w"],
                        lambda e: W.expert_slice(wts, e), lambda s: W.expert_slice(wts, s, shared=True))
    got = out.double().cpu().numpy()
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-2
