"""Shared helpers of the parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded bytes, and compare them by the rules the
layer fixes (exact routing except oracle-reported near-ties, exact
permutation, float tolerances)."""
from __future__ import annotations

import numpy as np
import torch

import expert_routing_grouped_layer_b200 as moe
import oracle
from expert_routing_grouped_layer_b200 import workloads as W

WEIGHT_REL_TOL = 1e-5  # top-k weights: fp32 against float64
LAYER_TOL = {"bf16": 1e-2, "fp8_e4m3_pow2_b128": 2e-2, "mxfp8": 2e-2,
             "nvfp4": 2e-2}  # rel-L2 of the output


def gpu_forward(cfg, inp, wts, T=None):
    """Run moe_layer_forward; return host copies of the output and intermediates."""
    T = cfg.T if T is None else T
    dev = inp["x"].device
    layer = moe.MoELayer(cfg, wts, inp["gate_w"], inp["gate_bias"], max_tokens=T, device=dev)
    x = inp["x"][:T].contiguous()
    out = layer.forward(x)
    torch.cuda.synchronize()
    k, E = cfg.num_experts_per_tok, cfg.n_routed_experts
    res = {
        "out": out.float().cpu().numpy().astype(np.float64),
        "idx": layer.intermediate(T, 0, torch.int32, (T, k)).cpu().numpy(),
        "w": layer.intermediate(T, 1, torch.float32, (T, k)).cpu().numpy(),
        "offsets": layer.intermediate(T, 2, torch.int32, (E + 1,)).cpu().numpy(),
        "sorted_pair": layer.intermediate(T, 3, torch.int32, (T * k,)).cpu().numpy(),
        "row_of": layer.intermediate(T, 4, torch.int32, (T * k,)).cpu().numpy(),
        "status": int(layer.status.item()),
    }
    del layer
    return res


def oracle_route(cfg, inp, tokens=None, T=None):
    T = cfg.T if T is None else T
    x = W.bf16_codes(inp["x"][:T])
    return oracle.route(cfg, x, inp["gate_w"].cpu().numpy(), inp["gate_bias"].cpu().numpy(),
                        tokens=tokens)


def compare_routing(cfg, g, r, tokens):
    """Expert sets equal and weights within tolerance for every token the oracle
    does not report as a near-tie, and the slot order (biased score descending)
    equal wherever the oracle does not report it as an order near-tie. Returns
    the number of near-tie tokens."""
    n_tie = 0
    otie = r.get("order_tie")
    for i, t in enumerate(tokens):
        if r["near_tie"][i]:
            n_tie += 1
            continue
        gi, oi = g["idx"][t], r["idx"][i]
        assert set(gi.tolist()) == set(oi.tolist()), "token %d: gpu %s oracle %s" % (t, gi, oi)
        if otie is not None and not otie[i]:
            assert np.array_equal(gi, oi), "token %d slot order: gpu %s oracle %s" % (t, gi, oi)
        gw = dict(zip(gi.tolist(), g["w"][t].tolist()))
        for e, w in zip(oi.tolist(), r["w"][i].tolist()):
            assert abs(gw[e] - w) <= WEIGHT_REL_TOL * abs(w), "token %d expert %d" % (t, e)
    return n_tie


def check_permutation_properties(cfg, g, T=None):
    """The GPU permutation is the stable expert-major sort of the GPU's own
    topk_idx: this fixes it uniquely, so checking these properties checks it
    exactly at any size."""
    T = cfg.T if T is None else T
    k, E = cfg.num_experts_per_tok, cfg.n_routed_experts
    flat = g["idx"].reshape(-1).astype(np.int64)
    N = T * k
    assert g["offsets"][0] == 0 and g["offsets"][E] == N
    assert np.array_equal(np.diff(g["offsets"]), np.bincount(flat, minlength=E))
    sp = g["sorted_pair"].astype(np.int64)
    assert np.array_equal(np.sort(sp), np.arange(N))
    assert np.array_equal(g["row_of"][sp], np.arange(N))
    assert np.array_equal(sp, np.argsort(flat, kind="stable"))


def oracle_layer_rows(cfg, inp, wts, idx, w, tokens):
    """Oracle output for the listed tokens with the oracle's own routing."""
    x = W.bf16_codes(inp["x"][torch.as_tensor(tokens, dtype=torch.long, device=inp["x"].device)])
    return oracle_layer(cfg, x, idx, w, wts)


def oracle_layer(cfg, x_codes, idx, w, wts):
    """The oracle's layer output for bf16 token rows given their routing, in the
    layer's weight format (NVFP4 layers: NVFP4 routed experts, bf16 shared)."""
    if cfg.wfmt == "nvfp4":
        return oracle.layer_nvfp4(cfg, x_codes, idx, w, lambda e: W.expert_slice(wts, e),
                                  lambda s: W.expert_slice(wts, s, shared=True),
                                  W.nvfp4_act_scales())
    return oracle.layer(cfg, x_codes, idx, w, lambda e: W.expert_slice(wts, e),
                        lambda s: W.expert_slice(wts, s, shared=True))


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def rel_l2_rows(a, b):
    """Relative L2 error of every row (token) separately."""
    return np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-300)


def compare_permutation_exact(cfg, g, r):
    """The GPU permutation against the oracle's (the oracle's stable sort of its
    own routing of every token), element by element, on the block of every
    expert that no near-tie token (by either side's choice) touches: the tokens
    of each block in order exactly, and each entry's pair index exactly unless
    that token's slot order is itself an oracle-reported near-tie. With no
    near-ties at all the offsets and the row_of inverse are compared whole.
    Returns the number of experts compared."""
    E, k = cfg.n_routed_experts, cfg.num_experts_per_tok
    off, sp, ro = oracle.permute(r["idx"], E)
    tie = np.nonzero(r["near_tie"])[0]
    otie = r.get("order_tie", np.zeros(len(r["near_tie"]), bool))
    touched = set(g["idx"][tie].ravel().tolist()) | set(r["idx"][tie].ravel().tolist())
    if tie.size == 0:
        assert np.array_equal(g["offsets"], off)
        if not otie.any():
            assert np.array_equal(g["sorted_pair"], sp)
            assert np.array_equal(g["row_of"], ro)
            return E
    n = 0
    for e in range(E):
        if e in touched:
            continue
        a = g["sorted_pair"][g["offsets"][e]:g["offsets"][e + 1]]
        b = sp[off[e]:off[e + 1]]
        assert np.array_equal(a // k, b // k), "expert %d: token order differs" % e
        keep = ~otie[b // k]
        assert np.array_equal(a[keep], b[keep]), "expert %d: slot indices differ" % e
        n += 1
    return n


def chosen_tokens(cfg, g, r, sample, seed):
    """Tokens whose layer output is checked one by one: a seeded random sample,
    plus tokens at the places where tiles end raggedly -- the first and last
    rows of the most loaded expert's block (its last, partial token tile), the
    rows of the least loaded non-empty expert (a one-token expert when there is
    one), the last rows of the last non-empty expert, and the first and last
    tokens (the shared experts' rows run in token order, so these sit in the
    shared segment's first and last tiles). Near-tie tokens are left out."""
    T, k = len(g["idx"]), cfg.num_experts_per_tok
    counts = np.diff(g["offsets"])
    sp = g["sorted_pair"]
    rows = []
    hot = int(counts.argmax())
    rows += [g["offsets"][hot], g["offsets"][hot + 1] - 2, g["offsets"][hot + 1] - 1]
    nz = np.nonzero(counts)[0]
    cold = int(nz[counts[nz].argmin()])
    rows += list(range(g["offsets"][cold], g["offsets"][cold + 1]))[:2]
    last = int(nz[-1])
    rows += [g["offsets"][last + 1] - 1]
    toks = {int(sp[x]) // k for x in rows if 0 <= x < len(sp)}
    toks |= {0, T - 1, max(0, T - 2)}
    rng = np.random.default_rng(seed)
    toks |= set(rng.choice(T, min(sample, T), replace=False).tolist())
    toks = np.array(sorted(t for t in toks if not r["near_tie"][t]), dtype=np.int64)
    return toks


def check_layer_tokens(cfg, inp, wts, g, r, toks, tol):
    """Per-token rel-L2 of the GPU output against the oracle (its own routing)
    on the listed tokens: the largest must be within tol. Returns the errors."""
    want = oracle_layer_rows(cfg, inp, wts, r["idx"][toks], r["w"][toks], toks)
    err = rel_l2_rows(g["out"][toks], want)
    assert err.max() <= tol, (float(err.max()), int(toks[err.argmax()]))
    return err
