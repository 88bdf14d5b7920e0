"""GPU parity of the quantised-weight / quantised-activation layers against the
float64 oracle (which decodes the same stored bytes), through the C ABI."""
import numpy as np
import pytest
import torch

import expert_routing_grouped_layer_b200 as moe
import oracle
from expert_routing_grouped_layer_b200 import workloads as W
from moe_testlib import (LAYER_TOL, check_permutation_properties, compare_routing, gpu_forward,
                         oracle_layer_rows, oracle_route, rel_l2)

pytestmark = pytest.mark.gpu


def _layer_check(cfg, T=None, sample=None, seed=0):
    T = cfg.T if T is None else T
    inp = W.make_inputs(cfg, "cuda")
    wts = W.make_weights(cfg, "cuda")
    g = gpu_forward(cfg, inp, wts, T)
    assert g["status"] == 0
    if sample is None:
        toks = np.arange(T)
        r = oracle_route(cfg, inp, T=T)
        rs = r
    else:
        toks = np.sort(np.random.default_rng(seed).choice(T, sample, replace=False))
        r = oracle_route(cfg, inp, T=T) if T <= 8192 else None
        rs = oracle_route(cfg, inp, tokens=toks.astype(np.int32), T=T)
    if r is not None:
        compare_routing(cfg, g, r, np.arange(T))
    else:
        compare_routing(cfg, g, rs, toks)
    check_permutation_properties(cfg, g, T)
    ok = ~rs["near_tie"]
    want = oracle_layer_rows(cfg, inp, wts, rs["idx"], rs["w"], toks)
    err = rel_l2(g["out"][toks][ok], want[ok])
    assert err <= LAYER_TOL[cfg.afmt], err
    return g, err


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
