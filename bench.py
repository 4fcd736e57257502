#!/usr/bin/env python3
"""Benchmark of the packed FP4 MoE layer (fe_moe) on B200.

Headline workload: a stack of 48 independent decode layers shaped like a
30B-A3B 128-expert model (E=128, H=2048, I=768, top-8, T=1 token), each with
its own seeded weights, x and router logits (seed 1000 + layer), run back to
back on one stream through the library's stack entry point
(fe_moe_stack_forward) and captured as one CUDA graph.  One step = one replay
= 48 layer forwards.  The stack touches
48 x 21.2 MB = 1.02 GB of expert weights per step, more than the 126 MB L2, so
no step finds its weights in L2 from the step before.

The other workloads of the layer run the same way, each as its own 48-layer
stack, and are reported in the same JSON line under "workloads": the T=64
decode batch with Zipf-skewed routing, the 512-expert layer at T=1 and T=4,
and the T=4096 prefill layer (a tensor-core roofline).

e2e: the same stack through fe_moe_stack_forward_host (the C-ABI call on host
buffers): every step copies all 48 layers' x and logits from pinned host
memory, runs the 48 layers and copies their y back.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
a bounded sample of the headline workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/s and achieved HBM GB/s (% of B200 peak) at T=1"
PREFILL_METRIC = "MoE-layer prefill tokens/s and tensor-core TFLOP/s at T=4096"
HEADLINE = "decode_e128_t1"
OTHERS = ["decode_e128_t64_zipf", "decode_e512_t1", "decode_e512_t4", "prefill_e128_t4096"]
NVFP4_WORKLOAD = "nvfp4_prefill_e128_t4096"
LAYERS = 48
NOMINAL_HBM_GBS = 8000.0
NOMINAL_FP4_TFLOPS = 9000.0
L2_BYTES = 126e6
PATH_NAMES = {1: "moderate-T path: routing + streaming mma.sync projections (sg_kernel) + ordered combine",
              2: "large-T path: routing + tensor-core tiles (tc_gemm_kernel) + ordered combine",
              3: "single-launch decode kernel (decode_kernel), one launch per layer"}


def kernel_label(path, launches_per_step, T):
    """What ran the step: the persistent stack kernel when the step was one launch per token."""
    if path == 3 and launches_per_step == T:
        return ("persistent stack kernel (stack_decode_kernel): every layer in one launch"
                + (" per token" if T > 1 else ""))
    return PATH_NAMES.get(path, str(path))
CSRC = os.path.join(ROOT, "fp4_expert_gemv_b200", "csrc")

# DRAM bytes (read + write) of a workload's dominant kernel come from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum), kept with the capture
# command and a hash of the kernel's source files in profiles/traffic.json.  They
# are reported only while those sources still hash to the captured value, null
# otherwise (the counters would describe another kernel).
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload, layers):
    """(DRAM bytes per launch of the kernel that runs all `layers` layers, kernel name), or
    (None, kernel) when the kernel changed since the capture, or (None, None)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, None
    with open(TRAFFIC_FILE) as f:
        entries = json.load(f).get("entries", [])
    for ent in entries:
        if ent.get("workload") != workload:
            continue
        if source_hash(ent["sources"]) != ent["sources_sha256_16"]:
            return None, ent["kernel"]
        return float(ent["dram_bytes_per_layer"]) * layers, ent["kernel"]
    return None, None


def bytes_per_expert(H, I):
    """Packed codes + bf16 group scales of one expert's gate_up and down matrices."""
    return (H // 2) * 2 * I + (H // 32) * 2 * I * 2 + (I // 2) * H + (I // 32) * H * 2


def algorithmic_bytes_per_layer(E, H, I, T, distinct_experts):
    """Touched experts' packed codes + scales, plus x, logits and y."""
    return distinct_experts * bytes_per_expert(H, I) + T * H * 2 + T * E * 4 + T * H * 2


def distinct_routed(logits, k):
    """Distinct experts the top-k of each row selects (ties to the lower index),
    by a host sort of the logits: used for the byte count only."""
    order = np.lexsort((np.broadcast_to(np.arange(logits.shape[-1]), logits.shape), -logits), axis=-1)
    return len(np.unique(order[:, :k]))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# --------------------------------------------------------------------------------------------

def oracle_sample_setup(cfg):
    """Layer 0 of the stack, token 0: the oracle's weights for its routed experts."""
    import oracle
    import synth
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    seed = synth.STACK_SEED0
    x = synth.activations_bf16(cfg["seeds"][0], 1, H)
    lg = synth.router_logits(seed, 1, E, cfg["zipf"])
    orc = oracle.default()
    idx, _ = orc.route(lg, k)
    ex = sorted(set(int(e) for e in idx.reshape(-1)))
    ew = orc.quantized_experts(E, synth.weights_gate_up(seed, E, H, I, experts=ex),
                               synth.weights_down(seed, E, I, H, experts=ex), ex)
    return orc, ew, x, lg, k


def time_oracle(cfg, reps: int):
    orc, ew, x, lg, k = oracle_sample_setup(cfg)
    orc.moe_forward(ew, x, lg, k)   # warm
    t0 = time.perf_counter()
    for _ in range(reps):
        orc.moe_forward(ew, x, lg, k)
    dt = time.perf_counter() - t0
    return dt / reps


def run_reference(args):
    world, rank, local = dist_setup()
    if rank != 0:
        return 0
    import synth
    cfg = synth.WORKLOADS[HEADLINE]
    orc, ew, x, lg, k = oracle_sample_setup(cfg)
    for _ in range(args.warmup):
        orc.moe_forward(ew, x, lg, k)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        orc.moe_forward(ew, x, lg, k)
        times.append(time.perf_counter() - t0)
    step_s = sum(times) / len(times)
    value = 1.0 / step_s
    sample = "layer 0 of the seeded stack, token 0 (8 experts), one single-threaded oracle forward per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
        "config": {"workload": HEADLINE, "E": cfg["E"], "H": cfg["H"], "I": cfg["I"], "top_k": cfg["top_k"],
                   "T": 1, "layers": 1, "parallelism": "cpu oracle, 1 thread"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------------------------

def build_stack(cfg, layers, device, max_T=None):
    """`layers` fe_moe handles with the seeded weights of seeds 1000 + l, drawn
    and packed on the device (the library's own packer)."""
    import torch

    import fp4_expert_gemv_b200 as fe
    import synth
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    st = torch.cuda.current_stream().cuda_stream
    handles = []
    Wgu = torch.empty((E, H, 2 * I), dtype=torch.float32, device=device)
    Wdn = torch.empty((E, I, H), dtype=torch.float32, device=device)
    gc = torch.empty((E, H // 2, 2 * I), dtype=torch.uint8, device=device)
    gs = torch.empty((E, H // 32, 2 * I), dtype=torch.int16, device=device)
    dc = torch.empty((E, I // 2, H), dtype=torch.uint8, device=device)
    ds = torch.empty((E, I // 32, H), dtype=torch.int16, device=device)
    for layer in range(layers):
        seed = synth.STACK_SEED0 + layer
        synth.device_gate_up(Wgu.data_ptr(), seed, E, H, I, st)
        synth.device_down(Wdn.data_ptr(), seed, E, I, H, st)
        fe.pack_device(Wgu, gc, gs)
        fe.pack_device(Wdn, dc, ds)
        m = fe.MoELayer(E, H, I, max_T=max_T or cfg["T"], max_top_k=k)
        m.load_packed(gc, gs, dc, ds)
        handles.append(m)
    torch.cuda.synchronize()
    del Wgu, Wdn, gc, gs, dc, ds
    torch.cuda.empty_cache()
    return handles


def stack_inputs(cfg, layers):
    """Every layer's seeded inputs (seed 1000 + l): x bf16 bits [layers, T, H]
    and router logits [layers, T, E]."""
    import synth
    T, H, E = cfg["T"], cfg["H"], cfg["E"]
    x = np.stack([synth.activations_bf16(synth.STACK_SEED0 + l, T, H) for l in range(layers)])
    lg = np.stack([synth.router_logits(synth.STACK_SEED0 + l, T, E, cfg["zipf"]) for l in range(layers)])
    return np.ascontiguousarray(x), np.ascontiguousarray(lg, dtype=np.float32)


def check_stack_parity(cfg, layers, x, lg, y_bits, check_layers, rows):
    """The timed graph's outputs of the given layers, on the given token rows,
    against the oracle (weights of seed 1000 + l), at the acceptance tolerance."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import harness
    import synth
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    out = {"rows": [int(r) for r in rows], "tolerance": {"max_rel": harness.MAX_REL_TOL, "l2_rel": harness.L2_REL_TOL},
           "layers": {}}
    ok = True
    for l in check_layers:
        osd = harness.OracleSide(E, H, I, synth.STACK_SEED0 + l)
        ref, _ = osd.forward(x[l][rows], lg[l][rows], k)
        mr, l2 = harness.output_errors(y_bits[l][rows], ref)
        good = bool(mr <= harness.MAX_REL_TOL and l2 <= harness.L2_REL_TOL)
        out["layers"][str(l)] = {"max_rel": mr, "l2_rel": l2, "ok": good}
        ok &= good
    out["ok"] = ok
    return out


def run_workload(name, args, device, world, rank, headline=False):
    """Build the workload's stack, time graph replays and the host-buffer call;
    returns a dict of measurements."""
    import torch

    import fp4_expert_gemv_b200 as fe
    import synth
    cfg = synth.WORKLOADS[name]
    E, H, I, k, T = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"], cfg["T"]
    layers = args.layers
    t_setup = time.perf_counter()
    handles = build_stack(cfg, layers, device)
    stack = fe.Stack(handles)
    setup_s = time.perf_counter() - t_setup

    x_host, lg = stack_inputs(cfg, layers)
    x_pin = torch.from_numpy(x_host.view(np.int16)).pin_memory()
    lg_pin = torch.from_numpy(lg).pin_memory()
    y_pin = torch.empty((layers, T, H), dtype=torch.int16).pin_memory()
    x_dev = x_pin.to(device).view(torch.bfloat16)
    lg_dev = lg_pin.to(device)
    y_dev = torch.empty((layers, T, H), dtype=torch.bfloat16, device=device)
    distinct = [distinct_routed(lg[l], k) for l in range(layers)]

    s = torch.cuda.Stream(device=device)
    with torch.cuda.stream(s):
        stack.forward(x_dev, lg_dev, k, y_dev, stream=s)
    torch.cuda.synchronize()
    path, kernels_per_layer = handles[0].last_forward_info()
    launches_per_step = stack.last_launches()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        stack.forward(x_dev, lg_dev, k, y_dev, stream=s)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    cur = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.nvtx.range_push(f"timed {name}")   # lets a profiler select the timed launches
    e0.record(cur)
    for i in range(args.steps):
        g.replay()
        step_ev[i].record(cur)   # per-step samples (median, min) besides the total
    e1.record(cur)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    # keep the GPU busy while the sampler catches the clocks of a loaded GPU
    t_extra = time.perf_counter()
    while time.perf_counter() - t_extra < 0.5:
        for _ in range(5):
            g.replay()
        torch.cuda.synchronize()
    clk = clocks.stop()
    ms_local = e0.elapsed_time(e1) / args.steps
    step_ms = [(e0 if i == 0 else step_ev[i - 1]).elapsed_time(step_ev[i]) for i in range(args.steps)]
    ms = max_over_ranks(ms_local, world, device)
    tokens_step = sum_over_ranks(layers * T, world, device)
    value = tokens_step / (ms / 1e3)

    # the same stack with one launch per layer (cross-layer streaming off; it applies
    # at T = 1): each layer then starts its weight stream when its own launch starts,
    # as a layer whose routing is only known once its own logits exist
    no_prefetch = None
    if T == 1:
        stack.set_prefetch(False)
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=s):
            stack.forward(x_dev, lg_dev, k, y_dev, stream=s)
        for _ in range(args.warmup):
            g2.replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0.record(cur)
        for _ in range(args.steps):
            g2.replay()
        e1.record(cur)
        torch.cuda.synchronize()
        ms2_local = e0.elapsed_time(e1) / args.steps
        ms2 = max_over_ranks(ms2_local, world, device)
        no_prefetch = {"ms_per_step": ms2, "us_per_layer": ms2_local * 1e3 / layers,
                       "value": tokens_step / (ms2 / 1e3), "unit": "tokens/s"}
        del g2
        stack.set_prefetch(True)

    # parity of the timed graph's outputs: layers 0 and 47 against the oracle
    parity = None
    if headline and not args.no_check:
        torch.cuda.synchronize()
        y_bits = y_dev.view(torch.int16).cpu().numpy().view(np.uint16)
        rows = np.arange(T) if T <= 8 else np.array([0, T // 2, T - 1])
        parity = check_stack_parity(cfg, layers, x_host, lg, y_bits, sorted({0, layers - 1}), rows)

    # end to end through the C ABI on host buffers (fe_moe_stack_forward_host):
    # H2D of x and every layer's logits, the layers, D2H of y, a stream sync
    h2d = x_pin.numel() * 2 + lg_pin.numel() * 4
    d2h = y_pin.numel() * 2
    for _ in range(3):
        stack.forward_host(x_pin, lg_pin, k, y_pin, stream=s)
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        stack.forward_host(x_pin, lg_pin, k, y_pin, stream=s)
    e2e_ms_local = (time.perf_counter() - t0) * 1e3 / args.steps
    e2e_ms = max_over_ranks(e2e_ms_local, world, device)
    e2e_value = tokens_step / (e2e_ms / 1e3)

    peaks, peak_kind = measured_peaks()
    bytes_layer = [algorithmic_bytes_per_layer(E, H, I, T, d) for d in distinct]
    bytes_step = float(sum(bytes_layer))
    us_layer = ms_local * 1e3 / layers
    traffic, traffic_kernel = ncu_traffic(name, layers) if launches_per_step == 1 else (None, None)
    prefill = name.startswith("prefill")
    if prefill:
        flops_layer = 2.0 * T * k * 3 * H * I
        tf = flops_layer * layers / (ms_local / 1e3) / 1e12
        tpeak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
        roofline = {"bound": "tensor", "achieved": tf, "peak": tpeak, "unit": "TFLOP/s", "frac": tf / tpeak,
                    "traffic": traffic, "kernel": kernel_label(path, launches_per_step, T),
                    "peak_kind": f"{peak_kind} sustained dense bf16 (f16 operands run at the same rate)",
                    "algorithmic_flops_per_layer": flops_layer,
                    "frac_of_nominal_fp4_9pflops": tf / NOMINAL_FP4_TFLOPS}
    else:
        achieved = bytes_step / (ms_local / 1e3) / 1e9
        if no_prefetch is not None:
            a2 = bytes_step / (no_prefetch["ms_per_step"] / 1e3) / 1e9
            no_prefetch["hbm_gbs"] = a2
            no_prefetch["frac"] = a2 / float(peaks["hbm_gbs"])
        roofline = {"bound": "hbm", "achieved": achieved, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                    "frac": achieved / float(peaks["hbm_gbs"]), "traffic": traffic,
                    "kernel": kernel_label(path, launches_per_step, T), "peak_kind": f"{peak_kind} HBM copy",
                    "algorithmic_bytes_per_layer_mean": bytes_step / layers,
                    "distinct_experts_per_layer_mean": float(np.mean(distinct)),
                    "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS}
    if traffic_kernel:
        roofline["traffic_kernel"] = traffic_kernel
        roofline["traffic_note"] = ("ncu dram__bytes_read.sum + dram__bytes_write.sum per layer of an "
                                    "8-layer capture x the layers of this launch (profiles/traffic.json)"
                                    if traffic is not None else "kernel changed since its ncu capture")
    res = {
        "workload": name, "E": E, "H": H, "I": I, "top_k": k, "T": T, "layers_per_step": layers,
        "steps": args.steps, "ms_per_step": ms, "us_per_layer": us_layer, "value": value,
        "unit": "tokens/s", "roofline": roofline, "clocks": clk,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "call": "fe_moe_stack_forward_host on pinned host buffers (every layer's x and logits in, y out; "
                        "synchronous)"},
        "gpu_launches": launches_per_step * args.steps,
        "launches_per_step": launches_per_step,
        "ms_per_step_median": float(np.median(step_ms)), "ms_per_step_min": float(np.min(step_ms)),
        "setup_s": setup_s,
        "l2": (f"inputs larger than L2: each step streams {layers} layers' routed experts ({bytes_step / 1e9:.2f} GB)"
               if bytes_step > L2_BYTES else
               f"step bytes ({bytes_step / 1e6:.0f} MB) fit in L2: not a valid HBM measurement"),
    }
    if parity is not None:
        res["parity"] = parity
    if no_prefetch is not None:
        res["one_launch_per_layer"] = no_prefetch
    if headline and not prefill_like(name):
        res["single_layer_l2_flushed"] = single_layer_flushed(handles[0], x_dev[0], lg_dev[0], k, y_dev[0],
                                                              bytes_layer[0], peaks)
    del g
    stack.close()
    for m in handles:
        m.close()
    del handles
    torch.cuda.empty_cache()
    return res


def prefill_like(name):
    return name.startswith("prefill")


def single_layer_flushed(layer, x, lg, k, y, nbytes, peaks, samples=40):
    """One layer (the stack's layer 0) as a one-forward CUDA graph, replayed with L2
    flushed between replays (a write of twice the L2 size, outside the timed events):
    median and min over the samples, after 10 warm-up replays."""
    import torch
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        layer.forward(x, lg, k, y, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        layer.forward(x, lg, k, y, stream=s)
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=x.device)
    for _ in range(10):
        g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(samples)]
    cur = torch.cuda.current_stream()
    for a, b in ev:
        flush.fill_(1)
        a.record(cur)
        g.replay()
        b.record(cur)
    torch.cuda.synchronize()
    us = np.array([a.elapsed_time(b) * 1e3 for a, b in ev])
    del g, flush
    med = float(np.median(us))
    gbs = nbytes / (med * 1e-6) / 1e9
    return {"us_median": med, "us_min": float(us.min()), "samples": samples,
            "kernel": "single-launch decode kernel (fe_moe_forward)",
            "achieved_gbs_at_median": gbs, "frac_of_measured_hbm": gbs / float(peaks["hbm_gbs"]),
            "l2": f"{2 * l2 / 1e6:.0f} MB written between replays, outside the timed events"}


def run_router(device):
    """The router GEMM fused with the top-k (fe_moe_router) on the decode layer's router
    (E 128, H 2048, top-8): at one token through 384 distinct W_r (192 MB, more than L2,
    so each call reads its W_r from HBM), and at 4096 tokens (a tensor-core GEMM),
    each timed over a CUDA graph of back-to-back calls."""
    import torch

    import fp4_expert_gemv_b200 as fe
    E, H, k = 128, 2048, 8
    peaks, src = measured_peaks()
    out = {}
    gen = torch.Generator(device=device)
    gen.manual_seed(4242)
    for T, n in ((1, 384), (4096, 16)):
        layer = fe.MoELayer(E, H, 64, T, k)
        wr = (torch.randn((n, E, H), generator=gen, device=device) / H ** 0.5).to(torch.bfloat16)
        x = torch.randn((T, H), generator=gen, device=device).to(torch.bfloat16)
        lg = torch.empty((n, T, E), dtype=torch.float32, device=device)
        idx = torch.empty((n, T, k), dtype=torch.int32, device=device)
        w = torch.empty((n, T, k), dtype=torch.float32, device=device)
        s = torch.cuda.Stream()

        def calls():
            for i in range(n):
                fe.check(fe.fe_moe_router(layer.h, x.data_ptr(), wr[i].data_ptr(), T, k, lg[i].data_ptr(),
                                          idx[i].data_ptr(), w[i].data_ptr(), s.cuda_stream), "fe_moe_router")

        with torch.cuda.stream(s):
            calls()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            calls()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(reps):
                g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (reps * n)
        st, bits = layer.status()
        rec = {"T": T, "E": E, "H": H, "top_k": k, "calls_per_graph": n, "us_per_call": us,
               "status_bits": bits, "splits_of_K": None}
        if T == 1:
            nbytes = E * H * 2 + T * H * 2 + T * E * 4 + T * k * 8
            gbs = nbytes / (us * 1e-6) / 1e9
            rec.update({"bound": "hbm", "algorithmic_bytes": nbytes, "achieved": gbs, "unit": "GB/s",
                        "peak": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"], "peak_source": src,
                        "note": "latency-bound at one token: 512 KB of W_r, one dependent chain of loads, "
                                "partial sums, the last CTA's sum and top-k"})
        else:
            flops = 2.0 * T * E * H
            tf = flops / (us * 1e-6) / 1e12
            rec.update({"bound": "tensor", "flops": flops, "achieved": tf, "unit": "TFLOP/s",
                        "peak": peaks["bf16_tflops"], "frac": tf / peaks["bf16_tflops"], "peak_source": src,
                        "note": "mma.sync bf16 tiles of 16 tokens x 8 experts; a small GEMM (2.1 GFLOP)"})
        del rec["splits_of_K"]
        out[f"T{T}"] = rec
        del g
        layer.close()
        del wr, x, lg, idx, w
        torch.cuda.empty_cache()
    return out


def int2_bytes_per_expert(H, I):
    """INT2 codes (2 bits) + bf16 group scales of one expert's gate_up and down matrices."""
    return (H // 4) * 2 * I + (H // 32) * 2 * I * 2 + (I // 4) * H + (I // 32) * H * 2


def run_int2(device, n_layers=16, steps=20):
    """The decode layer (E 128, H 2048, I 768, top-8, T = 1) with every odd expert held as
    INT2 codes (fe_moe_load_int2), 16 layers with their own seeded weights, x and logits
    (more bytes per step than L2 holds), one launch per layer in a CUDA graph; against the
    same 16 layers with every expert E2M1."""
    import torch

    import fp4_expert_gemv_b200 as fe
    import synth
    cfg = synth.WORKLOADS[HEADLINE]
    E, H, I, k, T = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"], cfg["T"]
    fmt = np.array([e % 2 for e in range(E)], dtype=np.uint8)
    handles = build_stack(cfg, n_layers, device)
    x, lg = stack_inputs(cfg, n_layers)
    st = torch.cuda.current_stream().cuda_stream
    peaks, src = measured_peaks()

    def timed():
        xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
        ld = torch.from_numpy(lg).to(device)
        yd = torch.empty_like(xd)
        s = torch.cuda.Stream()

        def calls():
            for l, m in enumerate(handles):
                fe.check(fe.fe_moe_forward(m.h, xd[l].data_ptr(), ld[l].data_ptr(), T, k, yd[l].data_ptr(),
                                           s.cuda_stream), "fe_moe_forward")

        with torch.cuda.stream(s):
            calls()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            calls()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(steps):
                g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1e3 / (steps * n_layers)

    us_fp4 = timed()
    Wgu = torch.empty((E, H, 2 * I), dtype=torch.float32, device=device)
    Wdn = torch.empty((E, I, H), dtype=torch.float32, device=device)
    for l, m in enumerate(handles):
        seed = synth.STACK_SEED0 + l
        synth.device_gate_up(Wgu.data_ptr(), seed, E, H, I, st)
        gc, gs = fe.pack_int2_device(Wgu)
        synth.device_down(Wdn.data_ptr(), seed, E, I, H, st)
        dc, ds = fe.pack_int2_device(Wdn)
        m.load_int2(fmt, gc, gs, dc, ds)
        del gc, gs, dc, ds
    del Wgu, Wdn
    us_mixed = timed()
    # algorithmic bytes: each layer's distinct routed experts in their own format, x, logits, y
    nbytes = 0.0
    for l in range(n_layers):
        order = np.lexsort((np.arange(E), -lg[l, 0].astype(np.float64)))
        for e in order[:k]:
            nbytes += int2_bytes_per_expert(H, I) if fmt[e] else bytes_per_expert(H, I)
        nbytes += T * H * 2 + T * E * 4 + T * H * 2
    per_layer = nbytes / n_layers
    gbs = per_layer / (us_mixed * 1e-6) / 1e9
    st_bits = [m.status()[1] for m in handles]
    for m in handles:
        m.close()
    torch.cuda.empty_cache()
    return {"workload": "decode_e128_t1, every odd expert INT2", "layers": n_layers, "T": T, "top_k": k,
            "us_per_layer": us_mixed, "tokens_per_s": T / (us_mixed * 1e-6),
            "algorithmic_bytes_per_layer_mean": per_layer,
            "roofline": {"bound": "hbm", "achieved": gbs, "unit": "GB/s", "peak": float(peaks["hbm_gbs"]),
                         "frac": gbs / float(peaks["hbm_gbs"]), "peak_source": src},
            "all_e2m1_us_per_layer": us_fp4,
            "path": "single-launch decode kernel, one launch per layer (the persistent kernel reads E2M1 only)",
            "status_bits": int(max(st_bits))}


def nvfp4_roofline(us_per_layer, T, k, H, I, peaks, src):
    """The block-scaled FP4 record's roofline: the layer's 2 T k (2 H I + I H) FLOPs per
    us_per_layer, against the measured sustained bf16 rate times 4 (the nominal FP4 : bf16
    ratio of the dense tensor peaks, 9 : 2.25 PFLOP/s)."""
    flops = 2.0 * T * k * (H * 2 * I + I * H)
    tf = flops / (us_per_layer * 1e-6) / 1e12
    fp4_peak = 4.0 * float(peaks["bf16_tflops_sustained"])
    return {"bound": "tensor", "achieved": tf, "unit": "TFLOP/s", "peak": fp4_peak, "frac": tf / fp4_peak,
            "frac_of_nominal_fp4_9pflops": tf / NOMINAL_FP4_TFLOPS,
            "peak_source": f"{src} bf16_tflops_sustained x 4 (nominal fp4 : bf16)"}


def run_nvfp4(device, n_layers=4, steps=8, warmup=3):
    """The prefill layer (E 128, H 2048, I 768, top-8, T = 4096) on the block-scaled FP4
    variant (fe_moe_load_nvfp4, FE_PATH_NVFP4): n_layers layers with their own seeded
    weights, x and logits (each layer's weight images alone exceed L2), one CUDA graph of
    the layers' forwards; the same layers on the exact tensor-core path beside it.  The
    variant approximates the layer (its distance to the exact layer is measured by the
    tests, not here)."""
    import torch

    import fp4_expert_gemv_b200 as fe
    import synth
    cfg = synth.WORKLOADS["prefill_e128_t4096"]
    E, H, I, k, T = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"], cfg["T"]
    st = torch.cuda.current_stream().cuda_stream
    handles = []
    Wgu = torch.empty((E, H, 2 * I), dtype=torch.float32, device=device)
    Wdn = torch.empty((E, I, H), dtype=torch.float32, device=device)
    for layer in range(n_layers):
        seed = synth.STACK_SEED0 + layer
        synth.device_gate_up(Wgu.data_ptr(), seed, E, H, I, st)
        synth.device_down(Wdn.data_ptr(), seed, E, I, H, st)
        gc, gs = fe.pack_device(Wgu)
        dc, ds = fe.pack_device(Wdn)
        m = fe.MoELayer(E, H, I, max_T=T, max_top_k=k)
        m.load_packed(gc, gs, dc, ds)
        m.load_nvfp4(gc, gs, dc, ds)
        handles.append(m)
        del gc, gs, dc, ds
    torch.cuda.synchronize()
    del Wgu, Wdn
    x, lg = stack_inputs(cfg, n_layers)
    xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    ld = torch.from_numpy(lg).to(device)
    yd = torch.empty_like(xd)
    peaks, src = measured_peaks()

    def timed(path):
        for m in handles:
            m.set_path(path)
        s = torch.cuda.Stream()

        def calls():
            for l, m in enumerate(handles):
                fe.check(fe.fe_moe_forward(m.h, xd[l].data_ptr(), ld[l].data_ptr(), T, k, yd[l].data_ptr(),
                                           s.cuda_stream), "fe_moe_forward")

        with torch.cuda.stream(s):
            calls()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            calls()
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(steps):
                g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1e3 / (steps * n_layers)

    us_nv = timed(fe.PATH_NVFP4)
    launches = handles[0].last_forward_info()[1]
    us_tc = timed(fe.PATH_TCGEN05)
    st_bits = [m.status()[1] for m in handles]
    for m in handles:
        m.close()
    del xd, ld, yd
    torch.cuda.empty_cache()
    return {"workload": "prefill_e128_t4096 on the block-scaled FP4 variant (NVFP4)", "layers": n_layers, "T": T,
            "top_k": k, "us_per_layer": us_nv, "tokens_per_s": T / (us_nv * 1e-6), "launches_per_layer": launches,
            "roofline": nvfp4_roofline(us_nv, T, k, H, I, peaks, src),
            "exact_tcgen05_us_per_layer": us_tc, "speedup_vs_exact_path": us_tc / us_nv,
            "accuracy": "an approximation of the layer: about 18 % l2 distance to the exact layer "
                        "(tests/test_gpu_nvfp4.py prints it per case)",
            "status_bits": int(max(st_bits))}


def run_gpu(args):
    import torch

    world, rank, local = dist_setup()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    head_name = HEADLINE if args.workload == "all" else args.workload
    others = [w for w in OTHERS if w != head_name] if args.workload == "all" else []

    head = run_workload(head_name, args, device, world, rank, headline=True)
    extra = {}
    for w in others:
        extra[w] = run_workload(w, args, device, world, rank)

    prefill = head_name.startswith("prefill")
    line = {
        "metric": PREFILL_METRIC if prefill else METRIC, "value": head["value"], "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded counter-based generator; random-init weights quantised to E2M1)",
        "config": {"workload": head_name, "E": head["E"], "H": head["H"], "I": head["I"], "top_k": head["top_k"],
                   "T": head["T"], "layers_per_step": head["layers_per_step"], "global_batch": head["T"] * world,
                   "parallelism": f"replicas x{world}", "l2": head["l2"],
                   "graph": f"one CUDA graph of fe_moe_stack_forward over {head['layers_per_step']} layers, "
                            "each with its own seeded weights, x and logits"},
        "us_per_layer": head["us_per_layer"],
        "roofline": head["roofline"],
        "clocks": head["clocks"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "setup_s": head["setup_s"],
    }
    if "parity" in head:
        line["parity"] = head["parity"]
    if "one_launch_per_layer" in head:
        line["one_launch_per_layer"] = head["one_launch_per_layer"]
    line["ms_per_step_median"] = head["ms_per_step_median"]
    line["ms_per_step_min"] = head["ms_per_step_min"]
    if "single_layer_l2_flushed" in head:
        line["single_layer_l2_flushed"] = head["single_layer_l2_flushed"]
    if extra:
        line["workloads"] = extra
    if args.workload == "all":
        line["router_gemm"] = run_router(device)
        line["int2_mixed"] = run_int2(device)
        line["nvfp4_prefill"] = run_nvfp4(device)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import synth
        reps = args.cpu_reps
        per = time_oracle(synth.WORKLOADS[head_name], reps) if not prefill else None
        if per is not None:
            line["cpu_baseline"] = {"value": 1.0 / per, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                    "sample": f"layer 0 of the stack, token 0, {reps} single-threaded oracle forwards"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fe", "reference"], default="fe")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--cpu-reps", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-check", action="store_true", help="skip the oracle check of the headline stack's output")
    ap.add_argument("--workload", default="all", choices=["all", HEADLINE] + OTHERS + [NVFP4_WORKLOAD],
                    help="all: the headline workload plus the others under 'workloads'; "
                         f"{NVFP4_WORKLOAD}: only the block-scaled FP4 variant's record (--layers layers, "
                         "--steps graph replays)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == NVFP4_WORKLOAD:
        import torch
        torch.cuda.set_device(0)
        rec = run_nvfp4(torch.device("cuda", 0), n_layers=min(args.layers, 8), steps=args.steps,
                        warmup=args.warmup)
        print(json.dumps(rec), flush=True)
        return 0
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
