"""B200 (sm_100a) routed mixture-of-experts layer forward.

Thin ctypes binding of ``libmoe.so`` (the C ABI in ``include/moe.h``). Every
function here only marshals arguments -- device pointers, sizes, the CUDA
stream -- and calls the library of the same name; all arithmetic runs in the
library's CUDA kernels. PyTorch provides device memory and streams only.

There is no fallback: if ``libmoe.so`` is missing, or no CUDA device is
present, every call raises. Build the library with
``python -m expert_routing_grouped_layer_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = range(5)
MOE_DEV_BAD_EXPERT = 1
MOE_DEV_TIMEOUT = 2

SCORE_FN = {"sigmoid": 0, "sqrtsoftplus": 1, "softmax": 2}
WFMT = {"bf16": 0, "fp8_e4m3_b128x128": 1, "fp4_e2m1_ue8m0_b32": 2, "mxfp4": 3, "nvfp4": 4}
AFMT = {"bf16": 0, "fp8_e4m3_pow2_b128": 1, "mxfp8": 2, "nvfp4": 3}

# symbols include/moe.h declares
EXPORTS = ("moe_workspace_bytes", "moe_gate_topk", "moe_permute", "moe_quantize_activations",
           "moe_pack_expert_inputs", "moe_expert_gate_up", "moe_expert_down",
           "moe_grouped_swiglu", "moe_combine", "moe_layer_forward", "moe_workspace_offset",
           "moe_status_string", "moe_permute_noalloc", "moe_selftest_wait_limit",
           "moe_rmsnorm_prologue", "moe_layer_forward_prenorm")

# capacity (int32 counts) of the static scratch behind moe_permute_noalloc
MOE_PERMUTE_NOALLOC_MAX_COUNTS = 262144

# moe_workspace_offset selectors
WS_TOPK_IDX, WS_TOPK_W, WS_OFFSETS, WS_SORTED_PAIR, WS_ROW_OF, WS_Y, WS_SHARED_Y, WS_XA, \
    WS_XA_SCALE, WS_H, WS_H_SCALE, WS_X_NORM = range(12)


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (where, _status_str(status), status))


class moe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_routed_experts", ctypes.c_int32),
                ("num_experts_per_tok", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("moe_intermediate_size", ctypes.c_int32),
                ("n_shared_experts", ctypes.c_int32), ("shared_intermediate_size", ctypes.c_int32),
                ("norm_topk_prob", ctypes.c_int32), ("routed_scaling_factor", ctypes.c_float),
                ("score_fn", ctypes.c_int32), ("wfmt", ctypes.c_int32), ("afmt", ctypes.c_int32),
                ("swiglu_limit", ctypes.c_float), ("nvfp4_x_scale", ctypes.c_float),
                ("nvfp4_h_scale", ctypes.c_float)]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w13", "w13_scale", "w2", "w2_scale", "sh_w13", "sh_w13_scale", "sh_w2",
                 "sh_w2_scale", "gate_w", "gate_bias", "w13_gscale", "w2_gscale")]


_lib = None
_lock = threading.Lock()
_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_I32 = ctypes.c_int32


def lib() -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    "libmoe.so is not built (expected at %s); run "
                    "`python -m expert_routing_grouped_layer_b200.build`" % LIB_PATH)
            l = ctypes.CDLL(LIB_PATH)
            CP = ctypes.POINTER(moe_config)
            WP = ctypes.POINTER(moe_weights)
            l.moe_workspace_bytes.restype = _SZ
            l.moe_workspace_bytes.argtypes = [CP, _I32]
            l.moe_workspace_offset.restype = _SZ
            l.moe_workspace_offset.argtypes = [CP, _I32, _I32]
            l.moe_selftest_wait_limit.restype = ctypes.c_int
            l.moe_selftest_wait_limit.argtypes = [_P, _P]
            l.moe_status_string.restype = ctypes.c_char_p
            l.moe_status_string.argtypes = [ctypes.c_int]
            l.moe_gate_topk.restype = ctypes.c_int
            l.moe_gate_topk.argtypes = [CP, _P, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]
            l.moe_permute.restype = ctypes.c_int
            l.moe_permute.argtypes = [CP, _P, _I32, _P, _P, _P, _P, _P, _SZ, _P]
            l.moe_permute_noalloc.restype = ctypes.c_int
            l.moe_permute_noalloc.argtypes = [CP, _P, _I32, _P, _P, _P, _P, _P]
            l.moe_quantize_activations.restype = ctypes.c_int
            l.moe_quantize_activations.argtypes = [CP, _P, _I32, _P, _P, _P]
            l.moe_pack_expert_inputs.restype = ctypes.c_int
            l.moe_pack_expert_inputs.argtypes = [CP, _P, _I32, _P, _P, _P, _P]
            l.moe_expert_gate_up.restype = ctypes.c_int
            l.moe_expert_gate_up.argtypes = [CP, _P, _P, _I32, _P, WP, _P, _P, _P, _P]
            l.moe_expert_down.restype = ctypes.c_int
            l.moe_expert_down.argtypes = [CP, _P, _P, _I32, _P, WP, _P, _P, _P, _P]
            l.moe_grouped_swiglu.restype = ctypes.c_int
            l.moe_grouped_swiglu.argtypes = [CP, _P, _I32, _P, _P, WP, _P, _P, _P, _SZ, _P, _P]
            l.moe_combine.restype = ctypes.c_int
            l.moe_combine.argtypes = [CP, _P, _P, _P, _P, _I32, _P, _P]
            l.moe_rmsnorm_prologue.restype = ctypes.c_int
            l.moe_rmsnorm_prologue.argtypes = [CP, _P, _I32, _P, ctypes.c_float, _P, _P, _P, _P]
            l.moe_layer_forward_prenorm.restype = ctypes.c_int
            l.moe_layer_forward_prenorm.argtypes = [CP, _P, _I32, _P, ctypes.c_float, WP, _P, _P,
                                                    _SZ, _P, _P]
            l.moe_layer_forward.restype = ctypes.c_int
            l.moe_layer_forward.argtypes = [CP, _P, _I32, WP, _P, _P, _SZ, _P, _P]
            _lib = l
    return _lib


def _status_str(s: int) -> str:
    try:
        return lib().moe_status_string(int(s)).decode()
    except Exception:
        return "status %d" % s


def _check(s: int, where: str):
    if s != MOE_OK:
        raise MoEError(s, where)


def _ptr(t) -> int | None:
    """Device address of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_config(cfg) -> moe_config:
    """moe_config from any object with the layer's field names (e.g. a MoEConfig)."""
    xs, hs = 1.0, 1.0
    if cfg.afmt == "nvfp4":
        xs, hs = getattr(cfg, "nvfp4_act_scales", None) or _nvfp4_act_scales()
    return moe_config(cfg.hidden, cfg.n_routed_experts, cfg.num_experts_per_tok, cfg.n_group,
                      cfg.topk_group, cfg.moe_intermediate_size, cfg.n_shared_experts,
                      cfg.shared_intermediate_size, int(bool(cfg.norm_topk_prob)),
                      float(cfg.routed_scaling_factor), SCORE_FN[cfg.score_fn], WFMT[cfg.wfmt],
                      AFMT[cfg.afmt], float(getattr(cfg, "swiglu_limit", 0.0)), float(xs),
                      float(hs))


def _nvfp4_act_scales():
    from . import workloads
    return workloads.nvfp4_act_scales()


def make_weights(w: dict, gate_w=None, gate_bias=None) -> moe_weights:
    g = lambda n: _ptr(w.get(n))
    return moe_weights(g("w13"), g("w13_scale"), g("w2"), g("w2_scale"), g("sh_w13"),
                       g("sh_w13_scale"), g("sh_w2"), g("sh_w2_scale"),
                       _ptr(gate_w if gate_w is not None else w.get("gate_w")),
                       _ptr(gate_bias if gate_bias is not None else w.get("gate_bias")),
                       g("w13_gscale"), g("w2_gscale"))


def _cfg(cfg):
    return cfg if isinstance(cfg, moe_config) else make_config(cfg)


# ----------------------------------------------------------------- entry points
def moe_workspace_bytes(cfg, T: int) -> int:
    return lib().moe_workspace_bytes(ctypes.byref(_cfg(cfg)), int(T))


def moe_workspace_offset(cfg, T: int, which: int) -> int:
    return lib().moe_workspace_offset(ctypes.byref(_cfg(cfg)), int(T), int(which))


def moe_gate_topk(cfg, x, T, gate_w, gate_bias, topk_idx, topk_w, ws, dev_status=None,
                  ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check(lib().moe_gate_topk(ctypes.byref(_cfg(cfg)), _ptr(x), int(T), _ptr(gate_w),
                               _ptr(gate_bias), _ptr(topk_idx), _ptr(topk_w), _ptr(dev_status),
                               _ptr(ws), ws_bytes, _stream(stream)), "moe_gate_topk")


def moe_permute(cfg, topk_idx, T, expert_offsets, sorted_pair, row_of, dev_status, ws,
                ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check(lib().moe_permute(ctypes.byref(_cfg(cfg)), _ptr(topk_idx), int(T), _ptr(expert_offsets),
                             _ptr(sorted_pair), _ptr(row_of), _ptr(dev_status), _ptr(ws), ws_bytes,
                             _stream(stream)), "moe_permute")


def moe_permute_noalloc(cfg, topk_idx, T, expert_offsets, sorted_pair, row_of, dev_status,
                        stream=None):
    """moe_permute without a workspace, for callers that may not allocate device
    memory: the library's own fixed 1 MiB device array holds the scratch.
    Raises MoEError (workspace too small) when ceil(T*k/4096) * n_routed_experts
    exceeds MOE_PERMUTE_NOALLOC_MAX_COUNTS. Concurrent calls race on that array."""
    _check(lib().moe_permute_noalloc(ctypes.byref(_cfg(cfg)), _ptr(topk_idx), int(T),
                                     _ptr(expert_offsets), _ptr(sorted_pair), _ptr(row_of),
                                     _ptr(dev_status), _stream(stream)), "moe_permute_noalloc")


def moe_quantize_activations(cfg, x, T, xq, xq_scale, stream=None):
    _check(lib().moe_quantize_activations(ctypes.byref(_cfg(cfg)), _ptr(x), int(T), _ptr(xq),
                                          _ptr(xq_scale), _stream(stream)),
           "moe_quantize_activations")


def moe_pack_expert_inputs(cfg, x, T, sorted_pair, xa, xa_scale, stream=None):
    _check(lib().moe_pack_expert_inputs(ctypes.byref(_cfg(cfg)), _ptr(x), int(T), _ptr(sorted_pair),
                                        _ptr(xa), _ptr(xa_scale), _stream(stream)),
           "moe_pack_expert_inputs")


def moe_expert_gate_up(cfg, xa, xa_scale, T, expert_offsets, weights, h, h_scale, dev_status,
                       stream=None):
    w = weights if isinstance(weights, moe_weights) else make_weights(weights)
    _check(lib().moe_expert_gate_up(ctypes.byref(_cfg(cfg)), _ptr(xa), _ptr(xa_scale), int(T),
                                    _ptr(expert_offsets), ctypes.byref(w), _ptr(h), _ptr(h_scale),
                                    _ptr(dev_status), _stream(stream)), "moe_expert_gate_up")


def moe_expert_down(cfg, h, h_scale, T, expert_offsets, weights, y, shared_y, dev_status,
                    stream=None):
    w = weights if isinstance(weights, moe_weights) else make_weights(weights)
    _check(lib().moe_expert_down(ctypes.byref(_cfg(cfg)), _ptr(h), _ptr(h_scale), int(T),
                                 _ptr(expert_offsets), ctypes.byref(w), _ptr(y), _ptr(shared_y),
                                 _ptr(dev_status), _stream(stream)), "moe_expert_down")


def moe_grouped_swiglu(cfg, x, T, sorted_pair, expert_offsets, weights, y, shared_y, ws,
                       dev_status, ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    w = weights if isinstance(weights, moe_weights) else make_weights(weights)
    _check(lib().moe_grouped_swiglu(ctypes.byref(_cfg(cfg)), _ptr(x), int(T), _ptr(sorted_pair),
                                    _ptr(expert_offsets), ctypes.byref(w), _ptr(y), _ptr(shared_y),
                                    _ptr(ws), ws_bytes, _ptr(dev_status), _stream(stream)),
           "moe_grouped_swiglu")


def moe_combine(cfg, y, shared_y, row_of, topk_w, T, out, stream=None):
    _check(lib().moe_combine(ctypes.byref(_cfg(cfg)), _ptr(y), _ptr(shared_y), _ptr(row_of),
                             _ptr(topk_w), int(T), _ptr(out), _stream(stream)), "moe_combine")


def moe_selftest_wait_limit(dev_status, stream=None):
    """Launch the wait-limit self-test: MOE_DEV_TIMEOUT lands in dev_status
    (device int32) about 2 s later, and the stream continues normally."""
    _check(lib().moe_selftest_wait_limit(_ptr(dev_status), _stream(stream)), "moe_selftest_wait_limit")


def moe_layer_forward(cfg, x, T, weights, out, ws, dev_status, ws_bytes=None, stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    w = weights if isinstance(weights, moe_weights) else make_weights(weights)
    _check(lib().moe_layer_forward(ctypes.byref(_cfg(cfg)), _ptr(x), int(T), ctypes.byref(w),
                                   _ptr(out), _ptr(ws), ws_bytes, _ptr(dev_status),
                                   _stream(stream)), "moe_layer_forward")


def moe_rmsnorm_prologue(cfg, x, T, norm_w, eps, x_norm, xq=None, xq_scale=None, stream=None):
    _check(lib().moe_rmsnorm_prologue(ctypes.byref(_cfg(cfg)), _ptr(x), int(T), _ptr(norm_w),
                                      float(eps), _ptr(x_norm), _ptr(xq), _ptr(xq_scale),
                                      _stream(stream)), "moe_rmsnorm_prologue")


def moe_layer_forward_prenorm(cfg, x, T, norm_w, eps, weights, out, ws, dev_status, ws_bytes=None,
                              stream=None):
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    w = weights if isinstance(weights, moe_weights) else make_weights(weights)
    _check(lib().moe_layer_forward_prenorm(ctypes.byref(_cfg(cfg)), _ptr(x), int(T), _ptr(norm_w),
                                           float(eps), ctypes.byref(w), _ptr(out), _ptr(ws),
                                           ws_bytes, _ptr(dev_status), _stream(stream)),
           "moe_layer_forward_prenorm")


class MoELayer:
    """A layer bound to its device-resident parameters and a workspace.

    ``forward(x)`` runs moe_layer_forward on the current stream and returns the
    bf16 output; ``x`` may live on the host (it is copied in first).
    """

    def __init__(self, cfg, weights: dict, gate_w, gate_bias, max_tokens: int, device="cuda"):
        import torch
        self.cfg = cfg
        self.ccfg = make_config(cfg)
        self.weights = weights
        self.gate_w, self.gate_bias = gate_w, gate_bias
        self.cw = make_weights(weights, gate_w, gate_bias)
        self.max_tokens = int(max_tokens)
        nbytes = moe_workspace_bytes(self.ccfg, self.max_tokens)
        if nbytes == 0:
            raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_bytes")
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.device = device

    def forward(self, x, out=None, stream=None):
        import torch
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError("more tokens than the workspace was sized for")
        if not x.is_cuda:
            x = x.to(self.device, non_blocking=True)
        if out is None:
            out = torch.empty(T, self.cfg.hidden, dtype=torch.bfloat16, device=self.device)
        moe_layer_forward(self.ccfg, x, T, self.cw, out, self.ws, self.status,
                          ws_bytes=self.ws.numel(), stream=stream)
        return out

    __call__ = forward

    def forward_prenorm(self, x, norm_w, eps, out=None, stream=None):
        """The layer from the un-normalised hidden state (moe_layer_forward_prenorm)."""
        import torch
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError("more tokens than the workspace was sized for")
        if out is None:
            out = torch.empty(T, self.cfg.hidden, dtype=torch.bfloat16, device=self.device)
        moe_layer_forward_prenorm(self.ccfg, x, T, norm_w, eps, self.cw, out, self.ws, self.status,
                                  ws_bytes=self.ws.numel(), stream=stream)
        return out

    def ws_ptr(self, T: int, which: int) -> int:
        """Device address of an intermediate inside the workspace."""
        return self.ws.data_ptr() + moe_workspace_offset(self.ccfg, T, which)

    def intermediate(self, T: int, which: int, dtype, shape):
        """A view of an intermediate left in the workspace by the last forward."""
        import torch
        off = moe_workspace_offset(self.ccfg, T, which)
        n = 1
        for s in shape:
            n *= s
        esz = torch.empty(0, dtype=dtype).element_size()
        return self.ws[off:off + n * esz].view(dtype).view(*shape)
