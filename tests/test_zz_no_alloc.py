"""moe_permute_noalloc: the permutation for callers that cannot allocate device
memory (a plugin inside a host runtime that owns all device allocations, or a
serving loop that may not enter the allocator) and so have no workspace to
pass. Its scratch is the library's own fixed device array. Checked through the
C ABI against moe_permute, which takes a caller workspace: the results are
integers and must match exactly, on two calls in a row (the second smaller, so
stale counts from the first would show)."""
import ctypes

import numpy as np
import pytest
import torch

import expert_routing_grouped_layer_b200 as moe
from expert_routing_grouped_layer_b200 import workloads as W


def _routing(T, k, E, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.rand(T, E, generator=g, device="cuda").argsort(dim=1)[:, :k].to(torch.int32)


def _with_workspace(cfg, idx, T):
    k, E = cfg.num_experts_per_tok, cfg.n_routed_experts
    ws = torch.empty(moe.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ro = torch.empty(T * k, dtype=torch.int32, device="cuda")
    moe.moe_permute(cfg, idx, T, off, sp, ro, st, ws)
    return off, sp, ro, st


def _no_alloc(cfg, idx, T):
    k, E = cfg.num_experts_per_tok, cfg.n_routed_experts
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    off = torch.full((E + 1,), -9, dtype=torch.int32, device="cuda")
    sp = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    ro = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    c = moe.make_config(cfg)
    s = moe.lib().moe_permute_noalloc(ctypes.byref(c), idx.data_ptr(), T, off.data_ptr(),
                                      sp.data_ptr(), ro.data_ptr(), st.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert s == moe.MOE_OK, moe.lib().moe_status_string(s)
    return off, sp, ro, st


@pytest.mark.gpu
def test_no_alloc_permute_matches_workspace_version_twice():
    cfg = W.CONFIGS["k2_decode_bf16"].replace(T=6000)  # several 4096-pair chunks
    k, E = cfg.num_experts_per_tok, cfg.n_routed_experts
    for T, seed in ((6000, 1), (1500, 2)):
        idx = _routing(T, k, E, seed)
        want = _with_workspace(cfg, idx, T)
        got = _no_alloc(cfg, idx, T)
        torch.cuda.synchronize()
        for a, b in zip(want, got):
            assert torch.equal(a, b)
        flat = idx.reshape(-1).cpu().numpy()
        assert np.array_equal(got[1].cpu().numpy(), np.argsort(flat, kind="stable"))


@pytest.mark.gpu
def test_no_alloc_permute_rejects_sizes_past_its_array():
    """One chunk past the array's limit is refused on the host before any launch.
    The buffers are real and full-sized, and topk_idx holds valid expert ids, so
    even a broken size check would only produce a wrong status, never a bad
    address."""
    cfg = W.CONFIGS["mx896"]  # 896 experts: the array holds 292 chunks of 4096 pairs
    k, E = cfg.num_experts_per_tok, cfg.n_routed_experts
    T = (moe.MOE_PERMUTE_NOALLOC_MAX_COUNTS // E + 1) * 4096 // k
    idx = _routing(T, k, E, 3)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    off = torch.full((E + 1,), -9, dtype=torch.int32, device="cuda")
    sp = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    ro = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    c = moe.make_config(cfg)
    s = moe.lib().moe_permute_noalloc(ctypes.byref(c), idx.data_ptr(), T, off.data_ptr(),
                                      sp.data_ptr(), ro.data_ptr(), st.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert s == moe.MOE_ERR_WORKSPACE
    with pytest.raises(moe.MoEError, match="workspace too small"):
        moe.moe_permute_noalloc(cfg, idx, T, off, sp, ro, st)
    torch.cuda.synchronize()
    # nothing was launched: every output still holds its fill value
    assert (off == -9).all() and (sp == -9).all() and (ro == -9).all() and st.item() == 0
