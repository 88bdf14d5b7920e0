"""The C-ABI library loads, exports every symbol include/moe.h declares, and
rejects bad arguments on the host before launching anything (these calls
never reach a kernel, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

import expert_routing_grouped_layer_b200 as moe
from expert_routing_grouped_layer_b200 import build as moe_build
from expert_routing_grouped_layer_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(moe.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_struct_layouts_match_header():
    assert ctypes.sizeof(moe.moe_config) == 16 * 4
    assert moe.moe_config.swiglu_limit.offset == 13 * 4  # appended after afmt
    assert moe.moe_config.nvfp4_h_scale.offset == 15 * 4
    assert ctypes.sizeof(moe.moe_weights) == 12 * 8


def cfg(**kw):
    return moe.make_config(W.CONFIGS["tiny_bf16"].replace(**kw))


BAD = [dict(hidden=100), dict(hidden=0), dict(n_routed_experts=0), dict(n_routed_experts=2048),
       dict(num_experts_per_tok=0), dict(num_experts_per_tok=33), dict(num_experts_per_tok=17),
       dict(n_group=3), dict(n_group=64, n_routed_experts=64), dict(topk_group=0),
       dict(n_group=4, topk_group=5), dict(n_group=8, topk_group=1, num_experts_per_tok=4),
       dict(moe_intermediate_size=100), dict(n_shared_experts=-1), dict(n_shared_experts=5),
       dict(norm_topk_prob=2), dict(routed_scaling_factor=0.0), dict(score_fn=7), dict(score_fn=3),
       dict(wfmt=9), dict(afmt=-1), dict(swiglu_limit=-1.0), dict(swiglu_limit=float("inf")),
       dict(swiglu_limit=float("nan"))]


@pytest.mark.parametrize("bad", BAD)
def test_invalid_configs_are_rejected(lib, bad):
    c = cfg()
    for k, v in bad.items():
        setattr(c, k, v)  # raw struct fields, as a C caller would pass them
    assert moe.moe_workspace_bytes(c, 64) == 0
    st = lib.moe_gate_topk(ctypes.byref(c), 16, 64, 16, 16, 16, 16, None, 16, 1 << 30, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    st = lib.moe_layer_forward(ctypes.byref(c), 16, 64, ctypes.byref(moe.moe_weights()), 16, 16,
                               1 << 30, None, None)
    assert st == moe.MOE_ERR_INVALID_ARG


def test_null_pointers_and_short_workspace_are_rejected(lib):
    c = cfg()
    need = moe.moe_workspace_bytes(c, 64)
    assert need > 0
    assert lib.moe_gate_topk(ctypes.byref(c), None, 64, 256, 256, 256, 256, None, 256, need,
                             None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_gate_topk(ctypes.byref(c), 256, 64, 256, 256, 256, 256, None, 256, 16,
                             None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_gate_topk(ctypes.byref(c), 8, 64, 256, 256, 256, 256, None, 256, need,
                             None) == moe.MOE_ERR_INVALID_ARG  # misaligned x
    assert lib.moe_permute(ctypes.byref(c), 256, 64, None, 256, 256, 256, 256, need, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(ctypes.byref(c), 256, 64, 256, 256, 256, 256, 256, 0, None) == \
        moe.MOE_ERR_WORKSPACE
    assert lib.moe_combine(ctypes.byref(c), None, 256, 256, 256, 64, 256, None) == \
        moe.MOE_ERR_INVALID_ARG
    w = moe.moe_weights()
    assert lib.moe_grouped_swiglu(ctypes.byref(c), 256, 64, 256, 256, ctypes.byref(w), 256, 256,
                                  256, need, None, None) == moe.MOE_ERR_INVALID_ARG
    w = moe.moe_weights(256, None, 256, None, 256, None, 256, None, 256, 256)
    assert lib.moe_layer_forward(ctypes.byref(c), 256, 64, ctypes.byref(w), 256, 256, need - 1,
                                 None, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_layer_forward(ctypes.byref(c), 256, -1, ctypes.byref(w), 256, 256, need, None,
                                 None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_quantize_activations(ctypes.byref(c), 256, 4, 256, 256, None) == \
        moe.MOE_ERR_INVALID_ARG  # bf16 activations have nothing to quantise


def test_zero_tokens_is_a_no_op(lib):
    c = cfg()
    w = moe.moe_weights()
    assert lib.moe_gate_topk(ctypes.byref(c), None, 0, None, None, None, None, None, None, 0,
                             None) == 0
    assert lib.moe_layer_forward(ctypes.byref(c), None, 0, ctypes.byref(w), None, None, 0, None,
                                 None) == 0


def test_unsupported_shared_width(lib):
    c = cfg(shared_intermediate_size=256)
    w = moe.moe_weights(256, None, 256, None, 256, None, 256, None, 256, 256)
    assert lib.moe_layer_forward(ctypes.byref(c), 256, 64, ctypes.byref(w), 256, 256, 1 << 40,
                                 None, None) == moe.MOE_ERR_UNSUPPORTED


def test_workspace_grows_with_tokens_and_offsets_fit(lib):
    for name in W.CONFIGS:
        c = moe.make_config(W.CONFIGS[name])
        a, b = moe.moe_workspace_bytes(c, 1), moe.moe_workspace_bytes(c, 4096)
        assert 0 < a < b
        T = W.CONFIGS[name].T
        total = moe.moe_workspace_bytes(c, T)
        k, H, S = W.CONFIGS[name].num_experts_per_tok, W.CONFIGS[name].hidden, \
            W.CONFIGS[name].n_shared_experts
        assert moe.moe_workspace_offset(c, T, 5) + T * k * H * 2 <= total
        assert moe.moe_workspace_offset(c, T, 6) + S * T * H * 2 <= total
        assert moe.moe_workspace_offset(c, T, 11) + T * H * 2 <= total  # x_norm
        assert moe.moe_workspace_offset(c, T, 12) == 2 ** 64 - 1


def test_fp8_weight_steps_need_h_scale_and_the_workspace_holds_it(lib):
    """With FP8 weights the gate/up call leaves h as f16 rows with one int8
    exponent per row in h_scale, which the down call reads: both reject a null
    h_scale before launching, and the workspace reserves N + S*T bytes for it."""
    base = W.CONFIGS["tiny_bf16"].replace(wfmt="fp8_e4m3_b128x128")
    c = moe.make_config(base)
    w = moe.moe_weights(256, 256, 256, 256, 256, 256, 256, 256, 256, 256)
    T = 64
    assert lib.moe_expert_gate_up(ctypes.byref(c), 256, 256, T, 256, ctypes.byref(w), 256, None,
                                  None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_down(ctypes.byref(c), 256, None, T, 256, ctypes.byref(w), 256, 256,
                               None, None) == moe.MOE_ERR_INVALID_ARG
    N, S = T * base.num_experts_per_tok, base.n_shared_experts
    total = moe.moe_workspace_bytes(c, T)
    hs = moe.moe_workspace_offset(c, T, 10)
    assert hs != 2 ** 64 - 1 and hs + N + S * T <= total


def test_prologue_arguments_are_checked_on_the_host(lib):
    """The RMSNorm prologue and the layer from the un-normalised hidden state
    reject bad eps, null or misaligned pointers and a short workspace before
    launching; quantised formats need their code and scale rows and H % 512.
    Every call here is refused (or has T = 0), so none reaches a kernel."""
    c = cfg()
    f = ctypes.c_float
    ok = lambda *a: lib.moe_rmsnorm_prologue(ctypes.byref(c), *a)
    assert ok(256, 64, 256, f(-1.0), 256, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert ok(256, 64, 256, f(float("inf")), 256, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert ok(256, 64, 256, f(float("nan")), 256, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert ok(None, 64, 256, f(1e-6), 256, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert ok(256, 64, 8, f(1e-6), 256, None, None, None) == moe.MOE_ERR_INVALID_ARG  # misaligned w
    assert ok(256, 0, None, f(1e-6), None, None, None, None) == moe.MOE_OK
    cq = cfg(afmt="mxfp8", wfmt="mxfp4", hidden=512, moe_intermediate_size=512,
             shared_intermediate_size=512)
    assert lib.moe_rmsnorm_prologue(ctypes.byref(cq), 256, 4, 256, f(1e-6), 256, None, 256,
                                    None) == moe.MOE_ERR_INVALID_ARG  # no code rows
    c256 = cfg(afmt="mxfp8", wfmt="mxfp4", hidden=256)
    assert lib.moe_rmsnorm_prologue(ctypes.byref(c256), 256, 4, 256, f(1e-6), 256, 256, 256,
                                    None) == moe.MOE_ERR_INVALID_ARG  # H % 512
    need = moe.moe_workspace_bytes(c, 64)
    w = moe.moe_weights(256, None, 256, None, 256, None, 256, None, 256, 256)
    lf = lambda *a: lib.moe_layer_forward_prenorm(ctypes.byref(c), *a)
    assert lf(256, 64, 256, f(1e-6), ctypes.byref(w), 256, 256, need - 1, None, None) == \
        moe.MOE_ERR_WORKSPACE
    assert lf(256, 64, None, f(1e-6), ctypes.byref(w), 256, 256, need, None, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert lf(256, 64, 256, f(-1e-6), ctypes.byref(w), 256, 256, need, None, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert lf(None, 0, None, f(1e-6), ctypes.byref(w), None, None, 0, None, None) == moe.MOE_OK


def test_status_strings(lib):
    assert moe.lib().moe_status_string(0) == b"ok"
    assert moe.lib().moe_status_string(3) == b"workspace too small"


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(moe, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        moe.lib()
