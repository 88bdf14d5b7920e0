"""The bench's accounting (CPU): algorithmic bytes and FLOPs in closed form for a
small layer, the binding-roof selection and the tensor peak per MMA class."""
import pytest

import bench
from expert_routing_grouped_layer_b200 import workloads as W

TINY = W.CONFIGS["tiny_bf16"]


def test_flops_closed_form():
    cfg = TINY.replace(T=40, hidden=256, moe_intermediate_size=128, num_experts_per_tok=4,
                       n_shared_experts=1)
    N = 40 * 4
    # each (token, expert) pair and each token through the shared expert: three H x I products
    assert bench.layer_flops(cfg, 40) == 2.0 * (N + 40) * 3 * 256 * 128
    assert bench.gate_up_flops(cfg, 40) == 2.0 * (N + 40) * 2 * 256 * 128


def test_bytes_closed_form_bf16():
    cfg = TINY.replace(T=40, hidden=256, moe_intermediate_size=128, num_experts_per_tok=4,
                       n_shared_experts=1, n_routed_experts=16)
    T, H, I, k, E, S, A = 40, 256, 128, 4, 16, 1, 9
    per_expert = 3 * H * I * 2  # bf16 W1, W3, W2
    assert bench.expert_bytes(cfg) == (per_expert, per_expert)
    assert bench.expert_weight_bytes(cfg, A) == (A + S) * per_expert
    # + router weight (fp32) + x read once + out written once (bf16)
    assert bench.layer_bytes(cfg, A, T) == (A + S) * per_expert + E * H * 4 + 2 * T * H * 2
    # gate/up: two thirds of the weights, the expert input rows, the intermediate rows
    N = T * k
    assert bench.gate_up_bytes(cfg, A, T) == pytest.approx(
        (A + S) * per_expert * 2 / 3 + (N + T) * H * 2 + (N + S * T) * I * 2)


def test_roofline_picks_the_binding_roof():
    hbm, tpeak = 6542.4, 1651.4
    # 1 GB and 1 GFLOP in 1 ms: HBM time 0.153 ms > tensor time 0.0006 ms
    r = bench.roofline(1e9, 1e9, 1.0, hbm, tpeak)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(1000.0) and r["frac"] == pytest.approx(1000.0 / hbm)
    # 1 MB and 1 TFLOP in 1 ms: tensor time 0.6 ms > HBM time 0.00015 ms
    r = bench.roofline(1e6, 1e12, 1.0, hbm, tpeak)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(1000.0) and r["frac"] == pytest.approx(1000.0 / tpeak)
    # both fractions are always reported
    assert r["hbm_frac"] == pytest.approx(1.0 / hbm) and r["tensor_frac"] == r["frac"]


def test_tensor_peak_per_mma_class():
    peaks = {"bf16_tflops": 1651.4}
    p, src = bench.tensor_peak(peaks, "measured", W.CONFIGS["k2_prefill_fp8w"])
    assert p == 1651.4 and src == "measured"  # FP8 weights with bf16 activations: f16 MMAs
    p, src = bench.tensor_peak(peaks, "measured", W.CONFIGS["v4_fp4"])
    assert p == pytest.approx(2 * 1651.4) and "nominal" in src  # block-scaled: FP8 rate


def test_decode_workload_is_hbm_bound_and_prefill_tensor_bound():
    peaks, src = bench.load_peaks()
    for name, active, bound in [("k2_decode_bf16", 160, "hbm"), ("k2_prefill_fp8w", 384, "tensor"),
                                ("v4_fp4", 384, "hbm"), ("mx896", 896, "tensor")]:
        cfg = W.CONFIGS[name]
        tp, _ = bench.tensor_peak(peaks, src, cfg)
        r = bench.roofline(bench.layer_bytes(cfg, active, cfg.T), bench.layer_flops(cfg, cfg.T), 1.0,
                           peaks["hbm_gbs"], tp)
        assert r["bound"] == bound, name


def test_clock_log_path():
    assert bench.clock_log_path(None, 3) is None
    assert bench.clock_log_path("c%d.csv", 3) == "c3.csv"
    assert bench.clock_log_path("c.csv", 3) == "c.csv"


@pytest.mark.parametrize("name,count", [("k2_decode_bf16", 9), ("k2_prefill_fp8w", 13),
                                        ("v4_fp4", 12), ("mx896", 11), ("k2_nvfp4", 14)])
def test_launch_count_matches_the_launch_lists(name, count):
    """The kernels one step of each workload launches on a 148-SM B200, as the
    ncu launch lists of the five workloads show them (one-kernel permutation up
    to 4096 pairs; two-pass packs; the FP8-weight h repack; the router's
    split-K reduction for the 8192- and 4096-token layers)."""
    cfg = W.CONFIGS[name]
    assert bench.launches_per_step(cfg, cfg.T, 148) == count


def test_tensor_peak_prefers_a_measured_fp8_rate():
    """Block-scaled layers take the best FP8 cuBLAS rate measured in the run;
    failed measurements (error strings) are ignored."""
    peaks = {"bf16_tflops": 1651.4}
    meas = {"fp8_e4m3_tensorwise": 3000.0, "mxfp8_block32": 3100.0,
            "nvfp4_block16_error": "not supported"}
    p, src = bench.tensor_peak(peaks, "measured", W.CONFIGS["v4_fp4"], meas)
    assert p == 3100.0 and "mxfp8_block32" in src
    # bf16-rate layers keep the bf16 figure
    p, _ = bench.tensor_peak(peaks, "measured", W.CONFIGS["k2_prefill_fp8w"], meas)
    assert p == 1651.4
    # NVFP4 layers take the NVFP4 rate, never an FP8 one
    p, src = bench.tensor_peak(peaks, "measured", W.CONFIGS["k2_nvfp4"],
                               dict(meas, nvfp4_block16=6000.0))
    assert p == 6000.0 and "nvfp4" in src
    p, src = bench.tensor_peak(peaks, "measured", W.CONFIGS["k2_nvfp4"], meas)
    assert p == pytest.approx(4 * 1651.4) and "nominal" in src


def test_roofline_flags_fractions_above_the_measured_peak():
    # 7 GB in 1 ms = 7000 GB/s: above the measured copy rate, below the datasheet
    r = bench.roofline(7e9, 1e9, 1.0, 6542.4, 1651.4)
    assert r["bound"] == "hbm" and r["above_measured_peak"]
    assert r["frac_of_nominal_hbm"] == pytest.approx(7000.0 / bench.NOMINAL_HBM_GBS)
    r = bench.roofline(6e9, 1e9, 1.0, 6542.4, 1651.4)
    assert not r["above_measured_peak"]


def test_both_arms_build_the_config_from_one_function():
    """The CUDA arm and the reference arm print the same config dict for a
    workload: both take it from workload_config, unchanged."""
    import inspect
    src = inspect.getsource(bench.measure) + inspect.getsource(bench.run_reference)
    assert src.count("workload_config(cfg, world)") == 2
    assert "cfgd[" not in src
    d = bench.workload_config(W.CONFIGS["mx896"], 1)
    assert d["T"] == 16384 and d["experts"] == 896 and d["weights"] == "mxfp4"


@pytest.mark.parametrize("T,E,H,splits", [(128, 384, 7168, 28), (8192, 384, 7168, 3),
                                          (4096, 384, 7168, 3), (16384, 896, 7168, 1),
                                          (64, 16, 256, 1), (700, 8, 512, 2)])
def test_router_split_plan(T, E, H, splits):
    """The router's K-split counts on 148 SMs, as measured best: every decode unit
    its own 4 k-blocks; three splits where one would leave a mostly idle second
    wave; none for the 896-expert layer (two measured slower)."""
    assert bench.router_splits(T, E, H, 148) == splits
