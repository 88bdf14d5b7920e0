"""Seeded synthetic workloads for the routed MoE layer.

This module only defines the layer configurations and draws their inputs. It
holds none of the layer's arithmetic (no routing, no permutation, no expert
math); both the CUDA path and the CPU oracle consume the bytes it produces.

Weight encoding here is the offline weight-preparation step (the pages'
convert.py / fp4_quant_kernel role): float weights drawn N(0, 0.02) are stored
in the format the layer reads. Which valid code a value rounds to is a property
of the input, not of the layer; both sides decode the stored bytes themselves.

Every tensor comes from a ``torch.Generator`` seeded with ``cfg.seed`` (plus a
fixed offset per tensor) on the device the caller names, so a workload is
reproducible per (seed, device type).

Layouts (row-major, leading index first):
  x            bf16  [T][H]                 post-attention-norm hidden states
  gate_w       fp32  [E][H]                 router weight
  gate_bias    fp32  [E]                    e_score_correction_bias
  w13          [E][2I][H]  rows 0..I-1 gate (W1), rows I..2I-1 up (W3)
  w2           [E][H][I]                    down projection
  sh_w13/sh_w2 the same with n_shared in place of E and I_sh in place of I
  bf16 weights: bfloat16 values.
  fp8_e4m3_b128x128: uint8 E4M3 codes + fp32 scale [mat][rows/128][cols/128].
  fp4_e2m1_ue8m0_b32 / mxfp4: uint8 packed E2M1 [mat][rows][cols/2] (even column
      in the low nibble) + uint8 E8M0 scale codes [mat][rows][cols/32].
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    hidden: int
    n_routed_experts: int
    num_experts_per_tok: int
    n_group: int
    topk_group: int
    moe_intermediate_size: int
    n_shared_experts: int
    shared_intermediate_size: int
    norm_topk_prob: bool
    routed_scaling_factor: float
    score_fn: str  # "sigmoid" | "sqrtsoftplus" | "softmax"
    wfmt: str  # "bf16" | "fp8_e4m3_b128x128" | "fp4_e2m1_ue8m0_b32" | "mxfp4" | "nvfp4"
    afmt: str  # "bf16" | "fp8_e4m3_pow2_b128" | "mxfp8" | "nvfp4"
    routing: str  # input recipe: "bias_uniform" | "balanced" | "zipf"
    seed: int
    description: str = ""
    swiglu_limit: float = 0.0  # 0: plain SwiGLU; L > 0: SiLU(min(g, L)) * clamp(u, -L, L)

    def replace(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    @property
    def n_pairs(self) -> int:
        return self.T * self.num_experts_per_tok


_SEED = 20261202

CONFIGS = {
    "tiny_bf16": MoEConfig(
        "tiny_bf16", T=64, hidden=256, n_routed_experts=16, num_experts_per_tok=4, n_group=1,
        topk_group=1, moe_intermediate_size=128, n_shared_experts=1, shared_intermediate_size=128,
        norm_topk_prob=True, routed_scaling_factor=2.827, score_fn="sigmoid", wfmt="bf16",
        afmt="bf16", routing="bias_uniform", seed=_SEED + 0,
        description="tiny layer, 16 experts top-4, bf16"),
    "k2_decode_bf16": MoEConfig(
        "k2_decode_bf16", T=128, hidden=7168, n_routed_experts=384, num_experts_per_tok=8,
        n_group=1, topk_group=1, moe_intermediate_size=2048, n_shared_experts=1,
        shared_intermediate_size=2048, norm_topk_prob=True, routed_scaling_factor=2.827,
        score_fn="sigmoid", wfmt="bf16", afmt="bf16", routing="bias_uniform", seed=_SEED + 1,
        description="Kimi-K2 / DeepSeek-V3 shaped decode layer, 128 tokens, bf16"),
    "k2_prefill_fp8w": MoEConfig(
        "k2_prefill_fp8w", T=8192, hidden=7168, n_routed_experts=384, num_experts_per_tok=8,
        n_group=8, topk_group=4, moe_intermediate_size=2048, n_shared_experts=1,
        shared_intermediate_size=2048, norm_topk_prob=True, routed_scaling_factor=2.827,
        score_fn="sigmoid", wfmt="fp8_e4m3_b128x128", afmt="bf16", routing="balanced",
        seed=_SEED + 2,
        description="same shape at prefill, 8192 tokens, group-limited 8/4, fp8 weights"),
    "v4_fp4": MoEConfig(
        "v4_fp4", T=4096, hidden=7168, n_routed_experts=384, num_experts_per_tok=6, n_group=1,
        topk_group=1, moe_intermediate_size=2048, n_shared_experts=1,
        shared_intermediate_size=2048, norm_topk_prob=True, routed_scaling_factor=2.5,
        score_fn="sqrtsoftplus", wfmt="fp4_e2m1_ue8m0_b32", afmt="fp8_e4m3_pow2_b128",
        routing="bias_uniform", seed=_SEED + 3,
        description="DeepSeek-V4 shaped, 4096 tokens, fp8 activations x fp4 experts"),
    "mx896": MoEConfig(
        "mx896", T=16384, hidden=7168, n_routed_experts=896, num_experts_per_tok=16, n_group=1,
        topk_group=1, moe_intermediate_size=1024, n_shared_experts=2,
        shared_intermediate_size=1024, norm_topk_prob=True, routed_scaling_factor=2.827,
        score_fn="sigmoid", wfmt="mxfp4", afmt="mxfp8", routing="zipf", seed=_SEED + 4,
        description="896 fine-grained experts top-16, 2 shared, MXFP8 x MXFP4, Zipf loads"),
    "k2_nvfp4": MoEConfig(
        "k2_nvfp4", T=4096, hidden=7168, n_routed_experts=384, num_experts_per_tok=8, n_group=1,
        topk_group=1, moe_intermediate_size=2048, n_shared_experts=1,
        shared_intermediate_size=2048, norm_topk_prob=True, routed_scaling_factor=2.827,
        score_fn="sigmoid", wfmt="nvfp4", afmt="nvfp4", routing="bias_uniform", seed=_SEED + 5,
        description="Kimi-K2 shaped, 4096 tokens, NVFP4 routed experts (W4A4, groups of 16 with "
                    "E4M3 scales), bf16 shared expert"),
}

# Input recipe constants (see the routing recipes in make_inputs).
BIAS_UNIFORM_HALF_WIDTH = 0.1  # e_score_correction_bias ~ U[-0.1, 0.1]
ROUTER_STD = 0.02  # router weight ~ N(0, 0.02)
WEIGHT_STD = 0.02  # expert weights ~ N(0, 0.02) before encoding
# balanced: logits carry a target component of this many router-row units on 8
# targets per token (2 experts in each of 4 groups, assigned cyclically so every
# expert is a target equally often); router weight drawn N(0, 0.004) so the
# random part of the logits (std ~0.34) rarely overturns a target; bias
# U[-0.005, 0.005]. Gives per-expert loads within about +7% / -10% of the mean.
BALANCED_TARGET_GAIN = 1.5
BALANCED_ROUTER_STD = 0.004
BALANCED_BIAS_HALF_WIDTH = 0.005
# zipf: bias_e = beta * ln(rank_e ** -1.1) over a seeded random rank order; with
# beta = 0.075 the sorted loads fall off with a fitted log-log slope near -1.1
# and the hottest expert takes well over 10x the mean.
ZIPF_S = 1.1
ZIPF_BETA = 0.075


def _gen(cfg: MoEConfig, device, offset: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed * 1000 + offset)
    return g


def make_inputs(cfg: MoEConfig, device="cpu"):
    """x (bf16 [T,H]), gate_w (fp32 [E,H]), gate_bias (fp32 [E]) for one config."""
    T, H, E = cfg.T, cfg.hidden, cfg.n_routed_experts
    dev = torch.device(device)
    g = _gen(cfg, dev, 1)
    if cfg.routing == "balanced":
        gate_w = torch.randn(E, H, generator=g, device=dev) * BALANCED_ROUTER_STD
        z = torch.randn(T, H, generator=g, device=dev)
        bias = (torch.rand(E, generator=g, device=dev) * 2 - 1) * BALANCED_BIAS_HALF_WIDTH
        ng, k = cfg.n_group, cfg.num_experts_per_tok
        gsz = E // ng
        per_group = 2
        n_groups_hit = k // per_group
        # random groups per token, then a cyclic walk through a shuffled order of
        # each group's experts so that every expert is targeted equally often
        grp = torch.rand(T, ng, generator=g, device=dev).argsort(dim=1)[:, :n_groups_hit]
        orders = torch.stack([torch.randperm(gsz, generator=g, device=dev) for _ in range(ng)])
        hit = torch.zeros(T, ng, dtype=torch.long, device=dev)
        hit.scatter_(1, grp, 1)
        occ = torch.cumsum(hit, dim=0) - 1  # occurrence index of each (token, group)
        counts = torch.zeros(T, E, device=dev)
        for q in range(per_group):
            o = torch.gather(occ, 1, grp) * per_group + q
            local = torch.gather(orders[grp], 2, (o % gsz).unsqueeze(2)).squeeze(2)
            counts.scatter_add_(1, grp * gsz + local, torch.ones_like(local, dtype=counts.dtype))
        unit = gate_w / (gate_w * gate_w).sum(dim=1, keepdim=True)
        x = z + BALANCED_TARGET_GAIN * (counts @ unit)
    else:
        x = torch.randn(T, H, generator=g, device=dev)
        gate_w = torch.randn(E, H, generator=g, device=dev) * ROUTER_STD
        if cfg.routing == "zipf":
            rank = torch.randperm(E, generator=g, device=dev).to(torch.float64) + 1.0
            bias = (ZIPF_BETA * torch.log(rank ** -ZIPF_S)).to(torch.float32)
        else:
            bias = (torch.rand(E, generator=g, device=dev) * 2 - 1) * BIAS_UNIFORM_HALF_WIDTH
    return {"x": x.to(torch.bfloat16).contiguous(), "gate_w": gate_w.float().contiguous(),
            "gate_bias": bias.float().contiguous()}


# Input recipe of the prologue (the post-attention RMSNorm in front of the
# layer): the hidden state before the norm is the workload's x with every row
# scaled by 2^u * (1 + v), u uniform on the integers -6..6 and v ~ U[0, 1), so
# rows span about four decades of magnitude; the norm weight is drawn
# N(1, 0.2) in fp32; eps = 1e-6.
PRENORM_EPS = 1e-6
PRENORM_WEIGHT_STD = 0.2


def make_prenorm_inputs(cfg: MoEConfig, x: torch.Tensor):
    """(x_resid bf16 [T,H], norm_w fp32 [H], eps) for the prologue, drawn from
    the workload's own x (same device) and the config's seed."""
    dev = x.device
    g = _gen(cfg, dev, 7)
    T, H = x.shape
    u = torch.randint(-6, 7, (T, 1), generator=g, device=dev).to(torch.float32)
    v = torch.rand(T, 1, generator=g, device=dev)
    x_resid = (x.float() * torch.exp2(u) * (1.0 + v)).to(torch.bfloat16).contiguous()
    norm_w = (1.0 + PRENORM_WEIGHT_STD * torch.randn(H, generator=g, device=dev)).float().contiguous()
    return x_resid, norm_w, PRENORM_EPS


# NVFP4 tensor scales of the routed experts' activations (calibration
# constants of the recipe): the input x ~ N(0,1) is covered up to |x| = 16 and
# the SwiGLU intermediate up to 128, i.e. g = amax / (6 * 448), so a group's
# scale code stays in E4M3's range with room to spare.
NVFP4_X_AMAX = 16.0
NVFP4_H_AMAX = 128.0


def nvfp4_act_scales():
    """(tensor scale of the experts' input, of their intermediate), fp32 values."""
    return (float(torch.tensor(NVFP4_X_AMAX / (6 * 448), dtype=torch.float32)),
            float(torch.tensor(NVFP4_H_AMAX / (6 * 448), dtype=torch.float32)))


# ------------------------------------------------------------- weight encoding
_E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _e2m1_codes(v: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 code (ties to the even code), saturating at +-6."""
    a = v.abs().clamp(max=6.0)
    grid = torch.tensor(_E2M1_GRID, device=v.device, dtype=a.dtype)
    dist = (a.unsqueeze(-1) - grid).abs()
    code = dist.argmin(dim=-1)  # first (lowest) code among equal distances
    nxt = (code + 1).clamp(max=7)
    d_here = torch.gather(dist, -1, code.unsqueeze(-1)).squeeze(-1)
    d_next = torch.gather(dist, -1, nxt.unsqueeze(-1)).squeeze(-1)
    code = torch.where(((code % 2) == 1) & (nxt != code) & (d_next == d_here), nxt, code)
    sign = (v < 0) & (code > 0)
    return (code + sign.to(code.dtype) * 8).to(torch.uint8)


def _pack_nibbles(codes: torch.Tensor) -> torch.Tensor:
    c = codes.reshape(*codes.shape[:-1], codes.shape[-1] // 2, 2)
    return (c[..., 0] | (c[..., 1] << 4)).contiguous()


def encode_weight(w: torch.Tensor, wfmt: str):
    """Encode float weights [mats][rows][cols] into (data, scale) for one format."""
    m, rows, cols = w.shape
    if wfmt == "bf16":
        return w.to(torch.bfloat16).contiguous(), None
    if wfmt == "fp8_e4m3_b128x128":
        blk = w.reshape(m, rows // 128, 128, cols // 128, 128)
        amax = blk.abs().amax(dim=(2, 4))
        scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).float()
        q = (blk / scale[:, :, None, :, None]).clamp(-448.0, 448.0)
        q = q.to(torch.float8_e4m3fn).view(torch.uint8).reshape(m, rows, cols)
        return q.contiguous(), scale.contiguous()
    if wfmt in ("fp4_e2m1_ue8m0_b32", "mxfp4"):
        blk = w.reshape(m, rows, cols // 32, 32).double()
        amax = blk.abs().amax(dim=3)
        safe = torch.where(amax > 0, amax, torch.ones_like(amax))
        if wfmt == "fp4_e2m1_ue8m0_b32":
            # power-of-two scale that brings the block into [-6, 6]
            e = torch.ceil(torch.log2(safe / 6.0))
            e = torch.where(safe > 6.0 * torch.exp2(e), e + 1, e)
            e = torch.where(safe <= 6.0 * torch.exp2(e - 1), e - 1, e)
        else:
            # OCP MX: 2^(floor(log2 amax) - 2), 2 = exponent of E2M1's largest power of two
            e = torch.frexp(safe)[1].double() - 1 - 2
        e = torch.where(amax > 0, e, torch.full_like(e, -127.0)).clamp(-127, 127)
        codes = _e2m1_codes((blk / torch.exp2(e)[..., None]).float()).reshape(m, rows, cols)
        return _pack_nibbles(codes), (e + 127).to(torch.uint8).contiguous()
    if wfmt == "nvfp4":
        # one fp32 tensor scale per matrix, g = amax / (6 * 448); per group of 16
        # an E4M3 scale code nearest amax_group / (6 g); E2M1 codes of w / (s g)
        blk = w.reshape(m, rows, cols // 16, 16).double()
        g = (blk.abs().amax(dim=(1, 2, 3)) / (6 * 448)).float()
        g = torch.where(g > 0, g, torch.ones_like(g))
        gd = g.double()[:, None, None]
        s = (blk.abs().amax(dim=3) / (6 * gd)).clamp(max=448).to(torch.float8_e4m3fn)
        sv = s.double()
        safe = torch.where(sv > 0, sv, torch.ones_like(sv))
        codes = _e2m1_codes((blk / (safe * gd)[..., None]).float())
        codes = torch.where((sv > 0)[..., None], codes, torch.zeros_like(codes)).reshape(m, rows, cols)
        return _pack_nibbles(codes), (s.view(torch.uint8).contiguous(), g.contiguous())
    raise ValueError("unknown weight format " + wfmt)


def make_weights(cfg: MoEConfig, device="cpu", experts=None):
    """Expert and shared-expert weights in cfg.wfmt.

    experts: optional iterable of routed expert ids to materialise; the others
    are left zero (their bytes are still allocated so layouts stay canonical).
    Each matrix is drawn from its own generator stream, so a matrix does not
    depend on which others are drawn.
    """
    dev = torch.device(device)
    H, E, I = cfg.hidden, cfg.n_routed_experts, cfg.moe_intermediate_size
    S, Ish = cfg.n_shared_experts, cfg.shared_intermediate_size

    def draw(offset, rows, cols):
        g = _gen(cfg, dev, offset)
        return torch.randn(1, rows, cols, generator=g, device=dev) * WEIGHT_STD

    out = {}
    for prefix, n_mat, inter, base in (("", E, I, 1000), ("sh_", S, Ish, 10_000_000)):
        which = range(n_mat) if (experts is None or prefix) else sorted(set(int(e) for e in experts))
        fmt = shared_wfmt(cfg) if prefix else cfg.wfmt
        for name, rows, cols, off in (("w13", 2 * inter, H, 0), ("w2", H, inter, 1)):
            data = scale = gscale = None
            for e in which:
                d, s = encode_weight(draw(base + 2 * e + off, rows, cols), fmt)
                g = None
                if isinstance(s, tuple):  # NVFP4: (group scale codes, tensor scale)
                    s, g = s
                if data is None:
                    data = torch.zeros((n_mat,) + tuple(d.shape[1:]), dtype=d.dtype, device=dev)
                    if s is not None:
                        scale = torch.zeros((n_mat,) + tuple(s.shape[1:]), dtype=s.dtype, device=dev)
                    if g is not None:
                        gscale = torch.ones(n_mat, dtype=torch.float32, device=dev)
                data[e] = d[0]
                if s is not None:
                    scale[e] = s[0]
                if g is not None:
                    gscale[e] = g[0]
            out[prefix + name] = data
            out[prefix + name + "_scale"] = scale
            if gscale is not None:
                out[prefix + name + "_gscale"] = gscale
    return out


def shared_wfmt(cfg: MoEConfig) -> str:
    """Weight format of the shared experts: the routed experts' format, except
    that NVFP4 layers keep them in bf16 (the NVFP4 recipe's exclusion list)."""
    return "bf16" if cfg.wfmt == "nvfp4" else cfg.wfmt


def weight_bytes_per_matrix(cfg: MoEConfig, inter: int, shared: bool = False) -> int:
    """Stored bytes (data + scales) of one expert's w13 plus w2 (a shared expert's
    when shared is set)."""
    P = 3 * cfg.hidden * inter
    fmt = shared_wfmt(cfg) if shared else cfg.wfmt
    if fmt == "bf16":
        return 2 * P
    if fmt == "nvfp4":
        return P // 2 + P // 16 + 8  # codes, group scales, two tensor scales
    if fmt == "fp8_e4m3_b128x128":
        return P + 4 * (P // (128 * 128))
    return P // 2 + P // 32


def expert_slice(weights: dict, e: int, shared: bool = False):
    """(w13, w13_scale, w2, w2_scale) of one matrix, as host numpy arrays with a
    leading dimension of 1 (bf16 returned as uint16 codes); NVFP4 routed experts
    add their two tensor scales (w13_gscale, w2_gscale) as a 6-tuple."""
    p = "sh_" if shared else ""

    def host(t):
        if t is None:
            return None
        t = t[e:e + 1].detach()
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
        a = t.cpu().numpy()
        return a.view("uint16") if a.dtype.name == "int16" else a

    out = (host(weights[p + "w13"]), host(weights[p + "w13_scale"]), host(weights[p + "w2"]),
           host(weights[p + "w2_scale"]))
    if weights.get(p + "w13_gscale") is not None:
        out = out + (host(weights[p + "w13_gscale"]), host(weights[p + "w2_gscale"]))
    return out


def bf16_codes(x: torch.Tensor):
    """Host uint16 codes of a bf16 tensor."""
    return x.detach().view(torch.int16).cpu().numpy().view("uint16")


def config_summary(cfg: MoEConfig) -> dict:
    return {k: v for k, v in dataclasses.asdict(cfg).items() if k != "description"}


__all__ = ["MoEConfig", "CONFIGS", "make_inputs", "make_prenorm_inputs", "make_weights",
           "encode_weight", "expert_slice",
           "bf16_codes", "weight_bytes_per_matrix", "config_summary"]

assert math.isclose(CONFIGS["k2_decode_bf16"].routed_scaling_factor, 2.827)
