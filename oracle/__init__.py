"""Float64 CPU oracle of the routed MoE layer forward pass.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package. It shares no code with the
CUDA library (``expert_routing_grouped_layer_b200``) and imports nothing from it;
configurations are read by attribute name only.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, one token or
one output element at a time); this module builds it with gcc, loads it with
ctypes and marshals numpy arrays. Every step cites its source passage there.

Pinned functions (each has ``-m "not gpu"`` tests against something other than
itself; see ``tests/test_oracle_*.py``): format decoders/encoders, the activation
quantisers, scoring, routing (brute force, library top-k, invariants), the
permutation (library stable argsort, bijection), one expert's SwiGLU (one-hot
closed forms, zero gate, linearity), the combine (identical-expert identity),
and the post-attention RMSNorm in front of the layer with its one-step
double -> bf16 rounding (brute force over the bf16 grid, a 60-digit evaluation
of the definition, closed forms, scale and permutation invariance).
The composed layer output has no worked example on the pages. It is pinned by
properties its definition fixes for any weights (each token's output depends on
that token alone; relabelling the experts changes nothing; the routed part
scales exactly with routed_scaling_factor; a common bias shift changes nothing),
with planted index mistakes shown to break them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SO = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

W_FMT = {"bf16": 0, "fp8_e4m3_b128x128": 1, "fp4_e2m1_ue8m0_b32": 2, "mxfp4": 3, "nvfp4": 4}
A_FMT = {"bf16": 0, "fp8_e4m3_pow2_b128": 1, "mxfp8": 2, "nvfp4": 3}
SCORE = {"sigmoid": 0, "sqrtsoftplus": 1, "softmax": 2}
NEAR_TIE_REL = 1e-6  # relative score gap under which a selection counts as a near-tie

_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            l = ctypes.CDLL(build())
            l.or_bf16_value.restype = _D
            l.or_bf16_value.argtypes = [ctypes.c_uint16]
            for f in ("or_e4m3_value", "or_e2m1_value", "or_e8m0_value"):
                getattr(l, f).restype = _D
                getattr(l, f).argtypes = [ctypes.c_uint8]
            l.or_e4m3_encode.restype = ctypes.c_uint8
            l.or_e4m3_encode.argtypes = [_D]
            l.or_pow2_ceil_exp.restype = _I
            l.or_pow2_ceil_exp.argtypes = [_D, _D]
            l.or_floor_log2.restype = _I
            l.or_floor_log2.argtypes = [_D]
            l.or_score.restype = _D
            l.or_score.argtypes = [_D, _I]
            l.or_quant_act.restype = _I
            l.or_quant_act.argtypes = [_I, _P, _I, _P, _P]
            l.or_dequant_act.restype = _I
            l.or_dequant_act.argtypes = [_I, _P, _P, _I, _P]
            l.or_weight_value.restype = _D
            l.or_weight_value.argtypes = [_I, _P, _P, _I, _I, _I, _I, _I]
            l.or_route_token.restype = _I
            l.or_route_token.argtypes = [_P, _D, _P, _P, _P, _D, _P, _P, _P, _P, _P, _P]
            l.or_route.restype = _I
            l.or_route.argtypes = [_P, _D, _P, _I, _P, _I, _P, _P, _D, _P, _P, _P, _P, _P]
            l.or_permute.restype = _I
            l.or_permute.argtypes = [_P, _I, _I, _I, _P, _P, _P]
            l.or_expert_input.restype = _I
            l.or_expert_input.argtypes = [_I, _P, _I, _I, _P, _P, _P]
            l.or_expert_rows.restype = _I
            l.or_expert_rows.argtypes = [_I, _I, _P, _P, _P, _P, _I, _I, _I, _P, _I, _D, _P]
            l.or_combine.restype = None
            l.or_combine.argtypes = [_I, _I, _I, _I, _P, _P, _P, _P]
            l.or_e2m1_encode.restype = ctypes.c_uint8
            l.or_e2m1_encode.argtypes = [_D]
            l.or_quant_nvfp4.restype = _I
            l.or_quant_nvfp4.argtypes = [_P, _I, _D, _P, _P]
            l.or_dequant_nvfp4.restype = _I
            l.or_dequant_nvfp4.argtypes = [_P, _P, _I, _D, _P]
            l.or_weight_value_nvfp4.restype = _D
            l.or_weight_value_nvfp4.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I]
            l.or_expert_rows_nvfp4.restype = _I
            l.or_expert_rows_nvfp4.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _I, _D, _D,
                                               _P]
            l.or_bf16_encode.restype = ctypes.c_uint16
            l.or_bf16_encode.argtypes = [_D, _D, _P]
            l.or_rmsnorm.restype = _I
            l.or_rmsnorm.argtypes = [_P, _I, _I, _P, _D, _D, _P, _P]
            _lib = l
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------- formats
def bf16_value(codes):
    l = lib()
    return np.array([l.or_bf16_value(int(c)) for c in np.ravel(codes)]).reshape(np.shape(codes))


def e4m3_value(codes):
    l = lib()
    return np.array([l.or_e4m3_value(int(c)) for c in np.ravel(codes)]).reshape(np.shape(codes))


def e2m1_value(codes):
    l = lib()
    return np.array([l.or_e2m1_value(int(c)) for c in np.ravel(codes)]).reshape(np.shape(codes))


def e8m0_value(codes):
    l = lib()
    return np.array([l.or_e8m0_value(int(c)) for c in np.ravel(codes)]).reshape(np.shape(codes))


def e4m3_encode(vals):
    l = lib()
    return np.array([l.or_e4m3_encode(float(v)) for v in np.ravel(vals)],
                    dtype=np.uint8).reshape(np.shape(vals))


def pow2_ceil_exp(amax: float, qmax: float) -> int:
    return lib().or_pow2_ceil_exp(float(amax), float(qmax))


def floor_log2(amax: float) -> int:
    return lib().or_floor_log2(float(amax))


def score(logit: float, score_fn: str) -> float:
    return lib().or_score(float(logit), SCORE[score_fn])


def quant_act(afmt: str, v):
    """Block-quantise one vector: returns (codes uint8[n], scale codes uint8[n/blk])."""
    v = _c(v, np.float64)
    n = v.shape[0]
    q = np.zeros(n, np.uint8)
    sc = np.zeros(max(1, n // 32), np.uint8)
    blk = lib().or_quant_act(A_FMT[afmt], _ptr(v), n, _ptr(q), _ptr(sc))
    if blk < 0:
        raise ValueError("bad activation format or length")
    return q, sc[: n // blk].copy()


def dequant_act(afmt: str, q, sc):
    q = _c(q, np.uint8)
    sc = _c(sc, np.uint8)
    out = np.zeros(q.shape[0], np.float64)
    if lib().or_dequant_act(A_FMT[afmt], _ptr(q), _ptr(sc), q.shape[0], _ptr(out)) < 0:
        raise ValueError("bad activation format or length")
    return out


def weight_value(wfmt: str, w, s, rows: int, cols: int, e: int, r: int, c: int) -> float:
    w = np.ascontiguousarray(w)
    s = None if s is None else np.ascontiguousarray(s)
    return lib().or_weight_value(W_FMT[wfmt], _ptr(w), _ptr(s), rows, cols, e, r, c)


def bf16_encode(vals, tie_rel: float = 0.0):
    """Round doubles to bf16 codes (RNE, one rounding); also returns the flags of
    values within tie_rel of a rounding midpoint."""
    l = lib()
    flat = np.ravel(np.asarray(vals, dtype=np.float64))
    codes = np.zeros(flat.shape, np.uint16)
    near = np.zeros(flat.shape, bool)
    f = ctypes.c_uint8(0)
    for i, v in enumerate(flat):
        codes[i] = l.or_bf16_encode(float(v), float(tie_rel), ctypes.byref(f))
        near[i] = bool(f.value)
    return codes.reshape(np.shape(vals)), near.reshape(np.shape(vals))


RMSNORM_TIE_REL = 2.0 ** -36  # a rounding near-tie: within this of a bf16 midpoint


def rmsnorm(x_u16, w, eps: float, tie_rel: float = RMSNORM_TIE_REL):
    """Post-attention RMSNorm of bf16 rows x [n, H] with fp32 weight w [H].

    Returns (out bf16 codes [n, H], near_tie bool [n, H])."""
    x = _c(x_u16, np.uint16)
    w = _c(w, np.float32)
    n, H = x.shape
    out = np.zeros((n, H), np.uint16)
    near = np.zeros((n, H), np.uint8)
    if lib().or_rmsnorm(_ptr(x), n, H, _ptr(w), float(eps), float(tie_rel), _ptr(out),
                        _ptr(near)) != 0:
        raise ValueError("bad RMSNorm arguments")
    return out, near.astype(bool)


def e2m1_encode(vals):
    """Round doubles to E2M1 codes (RNE, saturating at +-6)."""
    l = lib()
    return np.array([l.or_e2m1_encode(float(v)) for v in np.ravel(vals)],
                    dtype=np.uint8).reshape(np.shape(vals))


def quant_nvfp4(v, g: float):
    """NVFP4 quantisation of one vector with tensor scale g: (E2M1 codes uint8[n]
    one per byte, E4M3 scale codes uint8[n/16])."""
    v = _c(v, np.float64)
    n = v.shape[0]
    q = np.zeros(n, np.uint8)
    sc = np.zeros(max(1, n // 16), np.uint8)
    if lib().or_quant_nvfp4(_ptr(v), n, float(g), _ptr(q), _ptr(sc)) < 0:
        raise ValueError("bad NVFP4 length or tensor scale")
    return q, sc[: n // 16].copy()


def dequant_nvfp4(q, sc, g: float):
    q = _c(q, np.uint8)
    sc = _c(sc, np.uint8)
    out = np.zeros(q.shape[0], np.float64)
    if lib().or_dequant_nvfp4(_ptr(q), _ptr(sc), q.shape[0], float(g), _ptr(out)) < 0:
        raise ValueError("bad NVFP4 length")
    return out


def weight_value_nvfp4(w, s, g, rows: int, cols: int, e: int, r: int, c: int) -> float:
    w = np.ascontiguousarray(w, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    g = np.ascontiguousarray(g, np.float32)
    return lib().or_weight_value_nvfp4(_ptr(w), _ptr(s), _ptr(g), rows, cols, e, r, c)


def expert_input_nvfp4(x_rows_u16, g: float):
    """Rows of bf16 x as an NVFP4 expert sees them: (dequantised float64 [n,H],
    codes uint8 [n,H], scale codes uint8 [n,H/16])."""
    x = bf16_value_rows(x_rows_u16)
    n, H = x.shape
    q = np.zeros((n, H), np.uint8)
    sc = np.zeros((n, H // 16), np.uint8)
    xin = np.zeros((n, H), np.float64)
    for r in range(n):
        q[r], sc[r] = quant_nvfp4(x[r], g)
        xin[r] = dequant_nvfp4(q[r], sc[r], g)
    return xin, q, sc


def bf16_value_rows(x_rows_u16):
    """float64 values of bf16 codes (exact: a bf16 code is the top half of a float32)."""
    x = _c(x_rows_u16, np.uint16)
    return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def expert_rows_nvfp4(w13, w13s, g13, w2, w2s, g2, e: int, I: int, H: int, xin, ga2: float,
                      limit: float = 0.0):
    """SwiGLU of NVFP4 expert e on dequantised input rows xin [n, H] -> y [n, H];
    the intermediate is NVFP4-quantised with tensor scale ga2."""
    xin = _c(xin, np.float64)
    n = xin.shape[0]
    y = np.zeros((n, H), np.float64)
    a = [np.ascontiguousarray(t) for t in (w13, w13s, g13, w2, w2s, g2)]
    rc = lib().or_expert_rows_nvfp4(_ptr(a[0]), _ptr(a[1]), _ptr(_c(a[2], np.float32)), _ptr(a[3]),
                                    _ptr(a[4]), _ptr(_c(a[5], np.float32)), e, I, H, _ptr(xin), n,
                                    float(ga2), float(limit), _ptr(y))
    if rc != 0:
        raise ValueError("bad NVFP4 expert arguments")
    return y


# ----------------------------------------------------------------- config
def icfg(cfg) -> np.ndarray:
    return np.array([cfg.hidden, cfg.n_routed_experts, cfg.num_experts_per_tok, cfg.n_group,
                     cfg.topk_group, cfg.moe_intermediate_size, cfg.n_shared_experts,
                     cfg.shared_intermediate_size, int(bool(cfg.norm_topk_prob)),
                     SCORE[cfg.score_fn], W_FMT[cfg.wfmt], A_FMT[cfg.afmt]], dtype=np.int32)


# ----------------------------------------------------------------- routing
def route(cfg, x_u16, wg, bias, tokens=None, tie_rel: float = NEAR_TIE_REL):
    """Route tokens (all, or the listed ones). x_u16: [T, H] bf16 codes.

    Returns dict idx int32[n,k], w float64[n,k], near_tie bool[n], gap float64[n],
    order_gap float64[n] (smallest relative gap between consecutive slots' s') and
    order_tie bool[n] (order_gap below tie_rel: the slot order is a near-tie).
    """
    x_u16 = _c(x_u16, np.uint16)
    wg = _c(wg, np.float32)
    bias = _c(bias, np.float32)
    T = x_u16.shape[0]
    toks = None if tokens is None else _c(tokens, np.int32)
    n = T if toks is None else toks.shape[0]
    k = cfg.num_experts_per_tok
    idx = np.zeros((n, k), np.int32)
    w = np.zeros((n, k), np.float64)
    nt = np.zeros(n, np.uint8)
    gap = np.zeros(n, np.float64)
    og = np.zeros(n, np.float64)
    ic = icfg(cfg)
    rc = lib().or_route(_ptr(ic), float(cfg.routed_scaling_factor), _ptr(x_u16), T, _ptr(toks), n,
                        _ptr(wg), _ptr(bias), float(tie_rel), _ptr(idx), _ptr(w), _ptr(nt),
                        _ptr(gap), _ptr(og))
    if rc != 0:
        raise ValueError("oracle routing failed (code %d)" % rc)
    return {"idx": idx, "w": w, "near_tie": nt.astype(bool), "gap": gap, "order_gap": og,
            "order_tie": og < tie_rel}


def route_token(cfg, xrow_u16, wg, bias, tie_rel: float = NEAR_TIE_REL):
    """One token, also returning its float64 logits."""
    xrow_u16 = _c(xrow_u16, np.uint16)
    wg = _c(wg, np.float32)
    bias = _c(bias, np.float32)
    k, E = cfg.num_experts_per_tok, cfg.n_routed_experts
    idx = np.zeros(k, np.int32)
    w = np.zeros(k, np.float64)
    nt = np.zeros(1, np.uint8)
    gap = np.zeros(1, np.float64)
    logits = np.zeros(E, np.float64)
    og = np.zeros(1, np.float64)
    ic = icfg(cfg)
    rc = lib().or_route_token(_ptr(ic), float(cfg.routed_scaling_factor), _ptr(xrow_u16), _ptr(wg),
                              _ptr(bias), float(tie_rel), _ptr(idx), _ptr(w), _ptr(nt), _ptr(gap),
                              _ptr(logits), _ptr(og))
    if rc != 0:
        raise ValueError("oracle routing failed (code %d)" % rc)
    return {"idx": idx, "w": w, "near_tie": bool(nt[0]), "gap": float(gap[0]), "logits": logits,
            "order_gap": float(og[0]), "order_tie": bool(og[0] < tie_rel)}


def permute(idx, n_experts: int):
    """Stable expert-major permutation of the (token, slot) pairs.

    Returns (expert_offsets int32[E+1], sorted_pair int32[T*k], row_of int32[T*k]).
    """
    idx = _c(idx, np.int32)
    T, k = idx.shape
    off = np.zeros(n_experts + 1, np.int32)
    sp = np.zeros(T * k, np.int32)
    ro = np.zeros(T * k, np.int32)
    if lib().or_permute(_ptr(idx), T, k, n_experts, _ptr(off), _ptr(sp), _ptr(ro)) != 0:
        raise ValueError("expert id out of range")
    return off, sp, ro


# ----------------------------------------------------------------- experts
def expert_input(afmt: str, x_rows_u16):
    """Rows of the layer input as the experts see them (dequantised act quant).

    Returns (xin float64[n,H], q uint8[n,H] or None, sc uint8[n,H/blk] or None).
    """
    x = _c(x_rows_u16, np.uint16)
    n, H = x.shape
    xin = np.zeros((n, H), np.float64)
    q = sc = None
    if afmt != "bf16":
        blk = 128 if afmt == "fp8_e4m3_pow2_b128" else 32
        q = np.zeros((n, H), np.uint8)
        sc = np.zeros((n, H // blk), np.uint8)
    if lib().or_expert_input(A_FMT[afmt], _ptr(x), n, H, _ptr(xin), _ptr(q), _ptr(sc)) != 0:
        raise ValueError("bad activation format or hidden size")
    return xin, q, sc


def expert_rows(wfmt: str, afmt: str, w13, w13s, w2, w2s, e: int, I: int, H: int, xin,
                limit: float = 0.0):
    """SwiGLU of matrix e of the given weight tensors on rows xin[n, H] -> y[n, H];
    limit > 0 clamps the gate from above and the up projection to +-limit."""
    xin = _c(xin, np.float64)
    n = xin.shape[0]
    y = np.zeros((n, H), np.float64)
    w13 = np.ascontiguousarray(w13)
    w2 = np.ascontiguousarray(w2)
    w13s = None if w13s is None else np.ascontiguousarray(w13s)
    w2s = None if w2s is None else np.ascontiguousarray(w2s)
    rc = lib().or_expert_rows(W_FMT[wfmt], A_FMT[afmt], _ptr(w13), _ptr(w13s), _ptr(w2), _ptr(w2s),
                              e, I, H, _ptr(xin), n, float(limit), _ptr(y))
    if rc != 0:
        raise ValueError("bad expert arguments")
    return y


def combine(w, y, ys):
    """out[t] = sum_j w[t,j] y[t,j] + sum_s ys[s,t]; w [n,k], y [n,k,H], ys [S,n,H]."""
    w = _c(w, np.float64)
    y = _c(y, np.float64)
    ys = _c(ys, np.float64)
    n, k, H = y.shape
    out = np.zeros((n, H), np.float64)
    lib().or_combine(n, k, ys.shape[0], H, _ptr(w), _ptr(y), _ptr(ys), _ptr(out))
    return out


def layer_nvfp4(cfg, x_rows_u16, idx, w, get_expert, get_shared, act_gscales):
    """Layer output with NVFP4 routed experts ([V3] 四): get_expert(e) returns
    (w13, w13_scale, w2, w2_scale, g13, g2) of that one matrix (leading dimension
    1), act_gscales = (tensor scale of the experts' input, of their
    intermediate); the shared experts stay bf16 (the page's exclusion list) and
    read the bf16 input unquantised; get_shared(s) returns bf16 (w13, None, w2,
    None)."""
    H, I, Ish = cfg.hidden, cfg.moe_intermediate_size, cfg.shared_intermediate_size
    idx = np.asarray(idx)
    n, k = idx.shape
    ga13, ga2 = act_gscales
    xin, _, _ = expert_input_nvfp4(x_rows_u16, ga13)
    lim = float(getattr(cfg, "swiglu_limit", 0.0))
    y = np.zeros((n, k, H), np.float64)
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        w13, w13s, w2, w2s, g13, g2 = get_expert(int(e))
        y[rows, slots] = expert_rows_nvfp4(w13, w13s, g13, w2, w2s, g2, 0, I, H, xin[rows], ga2,
                                           lim)
    xb, _, _ = expert_input("bf16", x_rows_u16)
    ys = np.zeros((cfg.n_shared_experts, n, H), np.float64)
    for s_ in range(cfg.n_shared_experts):
        w13, _, w2, _ = get_shared(s_)
        ys[s_] = expert_rows("bf16", "bf16", w13, None, w2, None, 0, Ish, H, xb, lim)
    return combine(w, y, ys)


def layer(cfg, x_rows_u16, idx, w, get_expert, get_shared):
    """Layer output for n token rows given their routing (idx [n,k], w [n,k]).

    get_expert(e) / get_shared(s) return (w13, w13_scale, w2, w2_scale) holding
    that one matrix (leading dimension 1), so the caller may stream weights
    from wherever they live. Experts are visited in ascending id and each runs
    on the rows routed to it ([V3] 三.4 order); every output value is the
    float64 definition regardless of that visiting order.
    """
    H, I, Ish = cfg.hidden, cfg.moe_intermediate_size, cfg.shared_intermediate_size
    idx = np.asarray(idx)
    n, k = idx.shape
    xin, _, _ = expert_input(cfg.afmt, x_rows_u16)
    lim = float(getattr(cfg, "swiglu_limit", 0.0))
    y = np.zeros((n, k, H), np.float64)
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        w13, w13s, w2, w2s = get_expert(int(e))
        y[rows, slots] = expert_rows(cfg.wfmt, cfg.afmt, w13, w13s, w2, w2s, 0, I, H, xin[rows], lim)
    ys = np.zeros((cfg.n_shared_experts, n, H), np.float64)
    for s in range(cfg.n_shared_experts):
        w13, w13s, w2, w2s = get_shared(s)
        ys[s] = expert_rows(cfg.wfmt, cfg.afmt, w13, w13s, w2, w2s, 0, Ish, H, xin, lim)
    return combine(w, y, ys)
