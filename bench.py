#!/usr/bin/env python
"""Throughput of the routed MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one process per GPU)

A step is one pass of the whole layer (router + top-k, dispatch permutation,
expert input gather, gate/up + SwiGLU, down projection, combine) over one
batch of the workload's tokens, run through the library's C ABI. Inputs are
resident in HBM when the timed region starts. Each timed step calls the six
staged entry points back to back, with CUDA events at the step's ends and
around the gate/up call (the dominant kernel, whose duration the roofline
uses); between the other calls the layer's kernels follow one another with
programmatic dependent launch. The per-stage split comes from a separate pass
with events between every pair of calls. Multi-GPU runs are replicas
(weak scaling): every rank holds all experts and runs its own batch; there is
no data-path collective, only a barrier and a max over ranks of the timing.

Prints one JSON line on rank 0 (fields documented in the repository design
notes). ``--impl reference`` times the float64 CPU oracle instead, on a bounded
sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s on 1 B200; % of HBM roofline (decode) / tensor peak (prefill)"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "k2_decode_bf16"
L2_FLUSH_BYTES = 256 << 20  # > 2x the 126 MB L2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def router_splits(T, E, H, n_sms):
    """K splits of the router GEMM, as the library plans them: the count that
    minimises (waves of units) x (k-blocks per unit) plus T*E*8 bytes per split
    costed at 4 MB per k-block time, at least 4 k-blocks per split."""
    epad = (E + 127) // 128 * 128
    kb = H // 64
    base = (epad // 128) * ((T + 127) // 128)
    slab = T * E * 8.0 / 4.0e6
    best, best_cost = 1, float("inf")
    for s in range(1, max(1, kb // 4) + 1):
        kbps = (kb + s - 1) // s
        if (kb + kbps - 1) // kbps != s:
            continue
        waves = (base * s + n_sms - 1) // n_sms
        cost = waves * kbps + (s * slab if s > 1 else 0.0)
        if cost < best_cost - 1e-9:
            best, best_cost = s, cost
    kbps = (kb + best - 1) // best
    return (kb + kbps - 1) // kbps


def launches_per_step(cfg, T, n_sms):
    """Kernels one layer step launches, mirroring the library's launch rules:
    router plane split, router GEMM, its split-K reduction when K is split;
    top-k; the permutation (one kernel up to 4096 pairs, else count, scan and
    scatter); the expert-input pack (a gather of bf16 rows, or, for quantised
    activations and for the f16 rows of FP8 weights, the token rows converted
    once and then gathered); gate/up (FP8 weights: plus the in-place f16 repack
    of h); down; combine."""
    E, H = cfg.n_routed_experts, cfg.hidden
    N = T * cfg.num_experts_per_tok
    splits = router_splits(T, E, H, n_sms)
    router = 2 + (1 if splits > 1 else 0)
    permute = 1 if N <= 4096 else 3
    fp8w = cfg.wfmt == "fp8_e4m3_b128x128" and cfg.afmt == "bf16"
    if cfg.afmt == "nvfp4":  # quantise the token rows, gather; bf16 shared experts launch apart
        sh = 1 if cfg.n_shared_experts > 0 else 0
        return router + 1 + permute + 2 + (1 + sh) + (1 + sh) + 1
    if fp8w:
        pack = 2
    elif cfg.afmt == "bf16":
        pack = 1
    else:  # quantise the token rows once, gather when the scale rows are whole 16-byte vectors
        pack = 2 if (H // 32) % 16 == 0 else 1
    gate_up = 2 if fp8w else 1
    return router + 1 + permute + pack + gate_up + 1 + 1


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling runs)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override the routed expert count (small profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--clock-log", default=None,
                    help="keep the raw nvidia-smi samples here (%%d = device index)")
    ap.add_argument("--cpu-sample-tokens", type=int, default=128)
    ap.add_argument("--no-per-workload", action="store_true",
                    help="time only the headline workload (N=1 runs otherwise also time the "
                         "prefill-shaped workloads)")
    ap.add_argument("--per-workload-steps", type=int, default=20)
    ap.add_argument("--per-workload-cpu-tokens", type=int, default=12)
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int, enabled: bool = True, log_path=None):
        """log_path: where the raw samples go (kept); default a temporary file."""
        self.proc = None
        self.keep = log_path is not None
        if log_path is None:
            import tempfile
            fd, log_path = tempfile.mkstemp(prefix="moe_clocks_%d_" % dev_index, suffix=".csv")
            os.close(fd)
        self.path = log_path
        if not enabled:
            return
        import torch
        p = torch.cuda.get_device_properties(dev_index)
        bus = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", bus, "--query-gpu=" + self.FIELDS, "--format=csv,noheader",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1].split()[0]), float(parts[2].split()[0]),
                                 parts[4], parts[5:9]))
                except ValueError:
                    continue
        if not self.keep:
            os.remove(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        load = [r[0] for r in rows if r[0] > 600] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ accounting
def expert_bytes(cfg):
    """Bytes of one routed (and one shared) expert's stored weights."""
    from expert_routing_grouped_layer_b200 import workloads as W
    return (W.weight_bytes_per_matrix(cfg, cfg.moe_intermediate_size),
            W.weight_bytes_per_matrix(cfg, cfg.shared_intermediate_size, shared=True))


def gate_up_bytes(cfg, active, T):
    """Algorithmic bytes of one gate/up launch: the W1/W3 weights of every active
    expert and of the shared experts (each read once), the expert input rows
    (each read once) and the intermediate written once."""
    routed, shared = expert_bytes(cfg)
    frac = 2.0 / 3.0  # w13 holds 2 of the 3 H x I matrices
    abytes = {"bf16": 2, "nvfp4": 0.5 + 1 / 16}.get(cfg.afmt, 1)
    N = T * cfg.num_experts_per_tok
    S = cfg.n_shared_experts
    return (active * routed + S * shared) * frac + (N + T) * cfg.hidden * abytes + \
        (N + S * T) * cfg.moe_intermediate_size * abytes


def layer_bytes(cfg, active, T):
    """Algorithmic bytes of the whole layer: active experts' and shared experts'
    weights, the router weight, x read once and the output written once."""
    routed, shared = expert_bytes(cfg)
    return active * routed + cfg.n_shared_experts * shared + \
        cfg.n_routed_experts * cfg.hidden * 4 + 2 * T * cfg.hidden * 2


def expert_weight_bytes(cfg, active):
    """Stored weight bytes of the active routed experts and the shared experts."""
    routed, shared = expert_bytes(cfg)
    return active * routed + cfg.n_shared_experts * shared


def layer_flops(cfg, T):
    N = T * cfg.num_experts_per_tok
    return 2.0 * (N + T * cfg.n_shared_experts) * 3 * cfg.hidden * cfg.moe_intermediate_size


def gate_up_flops(cfg, T):
    """FLOPs of one gate/up launch: 2 of the 3 H x I products of every (token,
    expert) pair and of every token through each shared expert."""
    return layer_flops(cfg, T) * 2.0 / 3.0


# Nominal dense tensor rates relative to bf16 (context: the FP8 rate is the
# one the block-scaled E2M1 x E4M3 MMAs run at).
NOMINAL_RATE_VS_BF16 = {"bf16": 1.0, "fp8": 2.0, "fp4": 4.0}
NOMINAL_HBM_GBS = 7700.0  # B200 HGX datasheet figure, for context beside the measured copy rate


def measure_fp8_peaks(dev, n=8192, reps=10):
    """Measured FP8-rate tensor throughput of cuBLAS on this GPU (TFLOP/s, best of
    `reps` back-to-back n^3 products, CUDA events): E4M3 x E4M3 with per-tensor
    scales, and the block-scaled MXFP8 form (E8M0 scale per 32 elements) when
    this torch exposes it. These are library GEMMs used only as the denominator
    of the block-scaled layers' tensor fraction, the way the bf16 peak is."""
    import torch
    out = {}
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()  # column-major operand
    one = torch.ones((), device=dev)

    def best(fn):
        fn()
        torch.cuda.synchronize()
        t = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            t.append(e0.elapsed_time(e1))
        return 2.0 * n ** 3 / (min(t) / 1e3) / 1e12

    try:
        out["fp8_e4m3_tensorwise"] = best(
            lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16))
    except Exception as e:  # noqa: BLE001 - report why, keep the bench line
        out["fp8_e4m3_tensorwise_error"] = str(e).splitlines()[0][:160]
    try:
        a4 = torch.randint(0, 255, (n, n // 2), dtype=torch.uint8, device=dev).view(
            torch.float4_e2m1fn_x2)
        b4 = torch.randint(0, 255, (n, n // 2), dtype=torch.uint8, device=dev).view(
            torch.float4_e2m1fn_x2)
        s4 = torch.full((n * (n // 16),), 0x38, dtype=torch.uint8, device=dev).view(
            torch.float8_e4m3fn)
        out["nvfp4_block16"] = best(
            lambda: torch._scaled_mm(a4, b4.t(), scale_a=s4, scale_b=s4, out_dtype=torch.bfloat16))
        del a4, b4, s4
    except Exception as e:  # noqa: BLE001
        out["nvfp4_block16_error"] = str(e).splitlines()[0][:160]
    try:
        e8 = getattr(torch, "float8_e8m0fnu")
        sa = torch.full((n * (n // 32),), 127, dtype=torch.uint8, device=dev).view(e8)
        sb = torch.full((n * (n // 32),), 127, dtype=torch.uint8, device=dev).view(e8)
        out["mxfp8_block32"] = best(
            lambda: torch._scaled_mm(a, b, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16))
    except Exception as e:  # noqa: BLE001
        out["mxfp8_block32_error"] = str(e).splitlines()[0][:160]
    del a, b
    torch.cuda.empty_cache()
    return out


def tensor_peak(peaks, peak_src, cfg, fp8_measured=None):
    """(TFLOP/s, source) of the tensor rate the expert GEMMs run at: the
    measured bf16 figure for bf16/f16 MMAs; for FP8-rate MMAs the best measured
    FP8 cuBLAS rate when one was measured in this run, else the bf16 figure
    times the nominal ratio."""
    kind = "bf16" if cfg.afmt == "bf16" else ("fp4" if cfg.afmt == "nvfp4" else "fp8")
    if kind == "bf16":
        return peaks["bf16_tflops"], peak_src
    meas = {k: v for k, v in (fp8_measured or {}).items()
            if isinstance(v, float) and k.startswith("nvfp4") == (kind == "fp4")}
    if meas:
        name = max(meas, key=meas.get)
        return meas[name], "measured in this run: cuBLAS %s 8192^3, best of 10" % name
    ratio = NOMINAL_RATE_VS_BF16[kind]
    return peaks["bf16_tflops"] * ratio, "%s bf16 x nominal %s/bf16 ratio %g" % (peak_src, kind, ratio)


def roofline(bytes_, flops, ms, hbm, tpeak):
    """The binding roof (the larger of bytes / HBM and FLOPs / tensor peak) and the
    achieved fraction of it, with both fractions."""
    s = ms / 1e3
    hbm_frac = bytes_ / s / 1e9 / hbm
    tensor_frac = flops / s / 1e12 / tpeak
    if flops / (tpeak * 1e12) > bytes_ / (hbm * 1e9):
        r = {"bound": "tensor", "achieved": flops / s / 1e12, "peak": tpeak, "unit": "TFLOP/s",
             "frac": tensor_frac, "hbm_frac": hbm_frac, "tensor_frac": tensor_frac}
    else:
        # the measured peak is a read+write copy; a read-mostly stream can pass it,
        # so the fraction of the datasheet bandwidth is given beside it
        r = {"bound": "hbm", "achieved": bytes_ / s / 1e9, "peak": hbm, "unit": "GB/s",
             "frac": hbm_frac, "hbm_frac": hbm_frac, "tensor_frac": tensor_frac,
             "frac_of_nominal_hbm": bytes_ / s / 1e9 / NOMINAL_HBM_GBS,
             "nominal_hbm_gbs": NOMINAL_HBM_GBS}
    r["above_measured_peak"] = r["frac"] > 1.0
    return r


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("workload") != workload:
        return None
    h = hashlib.sha256()
    for src in e["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    return e["dram_bytes_per_launch"] if h.hexdigest()[:16] == e["source_sha256_16"] else None


# ------------------------------------------------------------------ ranks
def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank timing over all ranks (identity on a single process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(seed: int, rank: int) -> int:
    """Token seed of a replica: rank 0 runs the workload's own batch."""
    return seed if rank == 0 else seed + 7919 * rank


# ------------------------------------------------------------------ our arm
def clock_log_path(pattern, device_index):
    """The clock-sample file for one device: the pattern with %d replaced by the
    device index when it has one, else the pattern itself (None: a temporary file)."""
    if not pattern:
        return None
    return pattern % device_index if "%d" in pattern else pattern


def workload_config(cfg, world):
    """The config dict both arms print for a workload (identical keys and values)."""
    return {"workload": "%s: T=%d tokens, hidden %d, %d routed experts top-%d, intermediate %d, "
                        "%d shared, %s weights, %s activations"
                        % (cfg.name, cfg.T, cfg.hidden, cfg.n_routed_experts,
                           cfg.num_experts_per_tok, cfg.moe_intermediate_size,
                           cfg.n_shared_experts, cfg.wfmt, cfg.afmt),
            "T": cfg.T, "hidden": cfg.hidden, "experts": cfg.n_routed_experts,
            "top_k": cfg.num_experts_per_tok, "n_group": cfg.n_group,
            "topk_group": cfg.topk_group, "intermediate": cfg.moe_intermediate_size,
            "shared_experts": cfg.n_shared_experts, "score_fn": cfg.score_fn,
            "weights": cfg.wfmt, "activations": cfg.afmt, "routing": cfg.routing,
            "seed": cfg.seed, "parallelism": "replicas x%d" % world,
            "l2": "256 MiB write before every timed step, outside the timed events"}


def measure(args, cfg, rank, world, dev, steps, warmup, n_stage, n_e2e, workload_key,
            fp8_measured=None):
    """Time `steps` layer steps of one workload on this rank (staged ABI calls,
    L2 flushed before each), plus the per-stage split and the end-to-end form.
    Returns (line fields, inputs, weights)."""
    import torch
    import expert_routing_grouped_layer_b200 as moe
    from expert_routing_grouped_layer_b200 import workloads as W

    T, k, E, H, I, S = (cfg.T, cfg.num_experts_per_tok, cfg.n_routed_experts, cfg.hidden,
                        cfg.moe_intermediate_size, cfg.n_shared_experts)
    inp = W.make_inputs(cfg, dev)
    if rank > 0:  # replicas: same model, each rank its own tokens
        inp["x"] = W.make_inputs(cfg.replace(seed=replica_seed(cfg.seed, rank)), dev)["x"]
    wts = W.make_weights(cfg, dev)
    torch.cuda.synchronize()

    layer = moe.MoELayer(cfg, wts, inp["gate_w"], inp["gate_bias"], max_tokens=T, device=dev)
    ccfg, cw = layer.ccfg, layer.cw
    P = lambda which: layer.ws_ptr(T, which)
    ws, wsb, st = layer.ws, layer.ws.numel(), layer.status
    x = inp["x"]
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    def mark(ev, j):
        if ev[j] is not None:
            ev[j].record(stream)

    def step(ev):
        mark(ev, 0)
        moe.moe_gate_topk(ccfg, x, T, inp["gate_w"], inp["gate_bias"], P(moe.WS_TOPK_IDX),
                          P(moe.WS_TOPK_W), ws, st, wsb, stream=sp)
        mark(ev, 1)
        moe.moe_permute(ccfg, P(moe.WS_TOPK_IDX), T, P(moe.WS_OFFSETS), P(moe.WS_SORTED_PAIR),
                        P(moe.WS_ROW_OF), st, ws, wsb, stream=sp)
        mark(ev, 2)
        moe.moe_pack_expert_inputs(ccfg, x, T, P(moe.WS_SORTED_PAIR), P(moe.WS_XA),
                                   P(moe.WS_XA_SCALE), stream=sp)
        mark(ev, 3)
        moe.moe_expert_gate_up(ccfg, P(moe.WS_XA), P(moe.WS_XA_SCALE), T, P(moe.WS_OFFSETS), cw,
                               P(moe.WS_H), P(moe.WS_H_SCALE), st, stream=sp)
        mark(ev, 4)
        moe.moe_expert_down(ccfg, P(moe.WS_H), P(moe.WS_H_SCALE), T, P(moe.WS_OFFSETS), cw,
                            P(moe.WS_Y), P(moe.WS_SHARED_Y), st, stream=sp)
        mark(ev, 5)
        moe.moe_combine(ccfg, P(moe.WS_Y), P(moe.WS_SHARED_Y), P(moe.WS_ROW_OF), P(moe.WS_TOPK_W),
                        T, out, stream=sp)
        mark(ev, 6)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(7)]
    for _ in range(warmup):
        flush.zero_()
        step(mk())
    torch.cuda.synchronize()
    # the staged calls and moe_layer_forward must agree bit for bit
    ref = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(ref.view(torch.int16), out.view(torch.int16)), "staged != layer forward"
    assert st.item() == 0, "device status %d" % st.item()

    # per timed step: start, gate/up start, gate/up end, end
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    di = dev.index if dev.index is not None else 0
    clocks = ClockSampler(di, enabled=not args.no_clocks,
                          log_path=clock_log_path(args.clock_log, di))
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    for e in events:
        flush.zero_()  # L2 flush outside the timed events
        step([e[0], None, None, e[1], e[2], None, e[3]])
    torch.cuda.synchronize()
    wall = time.perf_counter() - t_wall
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[3]) for e in events]
    gate_up_ms = [e[1].elapsed_time(e[2]) for e in events]
    total_ms = max_over_ranks(sum(step_ms), dev)
    assert torch.equal(ref.view(torch.int16), out.view(torch.int16)), "timed steps changed output"

    # per-stage split: the staged entry points with events between them (not
    # part of the timed steps above)
    sevents = [mk() for _ in range(n_stage)]
    for i in range(n_stage):
        flush.zero_()
        step(sevents[i])
    torch.cuda.synchronize()
    stage = [[sevents[i][j].elapsed_time(sevents[i][j + 1]) for i in range(n_stage)]
             for j in range(6)]
    # the fused prologue (post-attention RMSNorm + activation quantisation) as its
    # own stage, on the workload's x scaled into an un-normalised hidden state
    xr, nw, eps = W.make_prenorm_inputs(cfg, x)
    xn = torch.empty_like(x)
    qa = cfg.afmt in ("fp8_e4m3_pow2_b128", "mxfp8")
    xq = torch.empty(T, H, dtype=torch.uint8, device=dev) if qa else None
    xqs = torch.empty(T, H // 32, dtype=torch.uint8, device=dev) if qa else None
    pro_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_stage)]
    for e0, e1 in pro_ev:
        flush.zero_()
        e0.record(stream)
        moe.moe_rmsnorm_prologue(ccfg, xr, T, nw, eps, xn, xq, xqs, stream=sp)
        e1.record(stream)
    torch.cuda.synchronize()
    pro_ms = statistics.fmean(e0.elapsed_time(e1) for e0, e1 in pro_ev)
    pro_bytes = 4 * T * H + ((T * H + T * H // 32) if qa else 0)
    del xr, xn, xq, xqs
    offsets = layer.intermediate(T, moe.WS_OFFSETS, torch.int32, (E + 1,)).cpu()
    counts = offsets[1:] - offsets[:-1]
    active = int((counts > 0).sum())

    # end to end: host tokens in (pinned), layer through the public API, host result out
    e2e = None
    if n_e2e > 0:
        xh = x.cpu().pin_memory()
        oh = torch.empty(T, H, dtype=torch.bfloat16).pin_memory()
        xd = torch.empty_like(x)
        for _ in range(3):
            xd.copy_(xh, non_blocking=True)
            oh.copy_(layer.forward(xd), non_blocking=True)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        # each step: L2 flushed first (outside the timed events), then the
        # pinned-host copy in, the layer, and the copy of the result back out
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_e2e)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record(stream)
            xd.copy_(xh, non_blocking=True)
            oh.copy_(layer.forward(xd), non_blocking=True)
            e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(statistics.fmean(e0.elapsed_time(e1) for e0, e1 in evs), dev)
        e2e = {"value": world * T / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2,
               "ms_per_step": e2e_ms, "includes_l2_flush": False}

    peaks, peak_src = load_peaks()
    ms = total_ms / steps
    mean = lambda j: statistics.fmean(stage[j])
    names = ["gate_topk", "permute", "pack_inputs", "gate_up", "down", "combine"]
    stage_ms = {n: mean(j) for j, n in enumerate(names)}
    gu_bytes = gate_up_bytes(cfg, active, T)
    gu_ms = statistics.fmean(gate_up_ms)  # the dominant kernel, over the timed steps
    hbm = peaks["hbm_gbs"]
    tpeak, tpeak_src = tensor_peak(peaks, peak_src, cfg, fp8_measured)
    lb = layer_bytes(cfg, active, T)
    lf = layer_flops(cfg, T)
    ewb = expert_weight_bytes(cfg, active)
    kroof = roofline(gu_bytes, gate_up_flops(cfg, T), gu_ms, hbm, tpeak)
    kroof.update({"kernel": "gate_up (grouped SwiGLU GEMM1)",
                  "peak_source": peak_src if kroof["bound"] == "hbm" else tpeak_src,
                  "traffic": ncu_traffic("gate_up", workload_key)
                  if not (args.tokens or args.experts) else None,
                  "algorithmic_bytes_per_launch": gu_bytes,
                  "algorithmic_flops_per_launch": gate_up_flops(cfg, T),
                  "ms_per_launch": gu_ms})
    lroof = roofline(lb, lf, ms, hbm, tpeak)
    lroof.update({"bytes": lb, "achieved_gbs": lb / (ms / 1e3) / 1e9,
                  # the activated and shared experts' weights alone (no router
                  # weight, no activations)
                  "expert_weight_bytes": ewb,
                  "expert_weight_frac": ewb / (ms / 1e3) / 1e9 / hbm,
                  "flops": lf, "tflops": lf / (ms / 1e3) / 1e12,
                  "tensor_peak": tpeak, "tensor_peak_source": tpeak_src})
    if cfg.afmt == "bf16":
        lroof["tensor_frac_sustained_peak"] = lf / (ms / 1e3) / 1e12 / peaks.get(
            "bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    cfgd = workload_config(cfg, world)
    routing_stats = {"active_experts": active,
                     "max_over_mean_load": float(counts.max()) / max(1e-9, float(counts.float().mean())),
                     "max_tokens_per_expert": int(counts.max())}
    fields = {
        "value": world * T / (ms / 1e3),
        "ms_per_step": ms,
        "steps": steps,
        "warmup": warmup,
        "dtype": "bf16" if cfg.wfmt == "bf16" else cfg.wfmt,
        "config": cfgd,
        "routing_stats": routing_stats,
        "roofline": kroof,
        "layer_roofline": lroof,
        "stage_ms": stage_ms,
        "prologue": {"kernel": "moe_rmsnorm_prologue (RMSNorm + act quant, one pass)",
                     "ms": pro_ms, "bytes": pro_bytes,
                     "achieved_gbs": pro_bytes / (pro_ms / 1e3) / 1e9,
                     "hbm_frac": pro_bytes / (pro_ms / 1e3) / 1e9 / load_peaks()[0]["hbm_gbs"],
                     "note": "not part of the timed layer step (the layer's input is the "
                             "normalised x); timed separately, L2 flushed before each call"},
        "stage_ms_source": "staged entry points with events between them, %d separate steps "
                           "(the timed steps record events only at their ends and around "
                           "gate_up)" % n_stage,
        "gpu_launches": launches_per_step(
            cfg, T, torch.cuda.get_device_properties(dev).multi_processor_count) * steps,
        "wall_s_timed_loop": wall,
        "clocks": clk,
        "e2e": e2e,
    }
    del layer, ws, out, flush, ref
    return fields, inp, wts


def cpu_baseline(cfg, inp, wts, tokens, seed=3):
    tok = min(tokens, cfg.T)
    times = oracle_timing(cfg, inp, wts, tok, 1, seed=seed)
    return {"value": tok / times[0], "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": "%d seeded tokens of the %d-token batch (route + layer, float64), %.1f s"
                      % (tok, cfg.T, times[0])}


# prefill-shaped workloads timed after the headline in an N=1 run
PER_WORKLOADS = ("k2_prefill_fp8w", "v4_fp4", "mx896", "k2_nvfp4")


def run_ours(args, rank, world, dev):
    import torch
    from expert_routing_grouped_layer_b200 import workloads as W

    cfg = W.CONFIGS[args.workload]
    if args.tokens:
        cfg = cfg.replace(T=args.tokens)
    if args.experts:
        cfg = cfg.replace(n_routed_experts=args.experts)
    fp8_measured = None
    if world == 1 and (cfg.afmt != "bf16" or not args.no_per_workload):
        fp8_measured = measure_fp8_peaks(dev)
    fields, inp, wts = measure(args, cfg, rank, world, dev, args.steps, args.warmup,
                               max(1, min(args.steps, 100)),
                               0 if args.no_e2e else max(1, min(args.steps, 100)),
                               args.workload, fp8_measured)
    line = {
        "metric": METRIC,
        "value": fields["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": fields["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": fields["dtype"],
        "data": "synthetic (seeded; x ~ N(0,1), router N(0,0.02), bias U[-0.1,0.1], "
                "experts N(0,0.02)); random-init weights",
    }
    line.update({k: v for k, v in fields.items() if k not in line})
    if fp8_measured is not None:
        line["fp8_peaks_tflops"] = fp8_measured
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, inp, wts, args.cpu_sample_tokens)
    del inp, wts
    torch.cuda.empty_cache()

    if world == 1 and not args.no_per_workload and not (args.tokens or args.experts):
        per = {}
        for name in PER_WORKLOADS:
            if name == args.workload:
                continue
            c = W.CONFIGS[name]
            f, inp, wts = measure(args, c, rank, world, dev, args.per_workload_steps,
                                  max(3, min(args.warmup, 5)), args.per_workload_steps,
                                  0 if args.no_e2e else min(args.per_workload_steps, 10),
                                  name, fp8_measured)
            keep = ("value", "ms_per_step", "steps", "warmup", "dtype", "config", "routing_stats",
                    "prologue", "roofline",
                    "layer_roofline", "stage_ms", "gpu_launches", "clocks", "e2e")
            per[name] = {k: f[k] for k in keep}
            per[name]["unit"] = UNIT
            if not args.no_cpu_baseline:
                per[name]["cpu_baseline"] = cpu_baseline(c, inp, wts,
                                                         args.per_workload_cpu_tokens)
            del inp, wts
            torch.cuda.empty_cache()
        line["per_workload"] = per
        line["per_workload_note"] = ("each prefill-shaped workload timed at full size after the "
                                     "headline, %d steps, same L2 flush and clock sampling; the "
                                     "headline value/config above is the decode workload"
                                     % args.per_workload_steps)
    return line


# ------------------------------------------------------------------ oracle arm
def oracle_timing(cfg, inp, wts, tokens_per_step, steps, seed=0):
    """Time the float64 oracle (route + layer) on `steps` disjoint samples of
    `tokens_per_step` tokens each; weights are fetched to host outside timing."""
    import numpy as np
    import oracle
    from expert_routing_grouped_layer_b200 import workloads as W

    rng = np.random.default_rng(seed)
    x_all = W.bf16_codes(inp["x"])
    wg = inp["gate_w"].cpu().numpy()
    bias = inp["gate_bias"].cpu().numpy()
    samples = [np.sort(rng.choice(cfg.T, tokens_per_step, replace=False)) for _ in range(steps)]
    cache = {}

    def get(e, shared=False):
        key = (e, shared)
        if key not in cache:
            cache[key] = W.expert_slice(wts, e, shared=shared)
        return cache[key]

    times = []
    for toks in samples:
        # routing first (timed), then fetch any expert not yet on the host (untimed)
        t0 = time.perf_counter()
        r = oracle.route(cfg, x_all, wg, bias, tokens=toks.astype(np.int32))
        t_route = time.perf_counter() - t0
        for e in np.unique(r["idx"]):
            get(int(e))
        for s in range(cfg.n_shared_experts):
            get(s, True)
        t0 = time.perf_counter()
        if cfg.wfmt == "nvfp4":
            oracle.layer_nvfp4(cfg, x_all[toks], r["idx"], r["w"], lambda e: get(e),
                               lambda s: get(s, True), W.nvfp4_act_scales())
        else:
            oracle.layer(cfg, x_all[toks], r["idx"], r["w"], lambda e: get(e),
                         lambda s: get(s, True))
        times.append(t_route + time.perf_counter() - t0)
        if len(cache) > 64:  # bound host memory
            cache.clear()
    return times


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, dev, world=1):
    import torch
    from expert_routing_grouped_layer_b200 import workloads as W
    cfg = W.CONFIGS[args.workload]
    inp = W.make_inputs(cfg, dev)
    wts = W.make_weights(cfg, dev)
    torch.cuda.synchronize()
    per_step = 1
    oracle_timing(cfg, inp, wts, per_step, args.warmup, seed=1)
    times = oracle_timing(cfg, inp, wts, per_step, args.steps, seed=2)
    total = sum(times)
    value = per_step * args.steps / total
    sample = "%d token(s) per step, %d steps, disjoint seeded samples of the %d-token batch" % (
        per_step, args.steps, cfg.T)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same workload as the CUDA arm)",
        "config": workload_config(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    import torch
    if args.impl == "reference":
        if rank != 0:
            return 0
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        print(json.dumps(run_reference(args, dev, world)), flush=True)
        return 0

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=dev,
                                             timeout=datetime.timedelta(seconds=300))
    line = run_ours(args, rank, world, dev)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
