#!/usr/bin/env python3
"""Benchmark of the packed FP4 MoE decode layer (fe_moe) on B200.

Workload: a stack of 48 independent decode layers shaped like a 30B-A3B
128-expert model (E=128, H=2048, I=768, top-8, T=1 token), each with its own
seeded weights (seed 1000 + layer), captured as one CUDA graph; the output of
layer l is the input of layer l+1, the router logits of every layer are
seeded inputs.  One step = one replay of the graph = 48 layer forwards.  The
stack touches 48 x 21.2 MB = 1.02 GB of expert weights per step, more than
the 126 MB L2, so no step finds its weights in L2 from the step before.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
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
WORKLOAD = "decode_e128_t1"
LAYERS = 48
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126e6
KERNEL_NAMES = {1: "streaming mma.sync projections sg_kernel (routing, gate_up, down, combine)",
                2: "tensor-core tiles tc_gemm_kernel (gate_up + down) with routing, row conversion and combine",
                3: "decode_kernel (whole layer, one cooperative launch); per-launch time = step time / layers"}
PREFILL_METRIC = "MoE-layer prefill tokens/s and tensor-core TFLOP/s at T=4096"
# DRAM bytes (read + write) per launch of the dominant kernel, from the ncu
# captures summarised in profiles/ (recaptured whenever that kernel changes)
TRAFFIC = {"decode_e128_t1": (21379072, "decode_kernel", "profiles/decode_kernel_decode_e128_t1.md"),
           "prefill_e128_t4096": (299220224, "tc_gemm_kernel gate_up", "profiles/tc_gemm_kernel_prefill_e128_t4096.md"),
           "decode_e128_t64_zipf": (95570432, "sg_kernel gate_up", "profiles/sg_kernel_decode_e128_t64_zipf.md")}
BYTES_PER_EXPERT = lambda H, I: (H // 2) * 2 * I + (H // 32) * 2 * I * 2 + (I // 2) * H + (I // 32) * H * 2  # noqa: E731


def algorithmic_bytes_per_layer(E, H, I, T, distinct_experts):
    """Touched experts' packed codes + scales, plus x, logits and y."""
    return distinct_experts * BYTES_PER_EXPERT(H, I) + T * H * 2 + T * E * 4 + T * H * 2


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s sustained under the power cap (the f16 tensor-core
    rate is the same): the denominator for a kernel timed inside a long step."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured sustained bf16 (f16 operands)"
    return 1400.0, "fallback sustained bf16"


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


# --------------------------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# --------------------------------------------------------------------------------------------

def oracle_sample_setup(cfg):
    """Layer 0 of the stack, token 0: the oracle's weights for its 8 experts."""
    import oracle
    import synth
    E, H, I, k = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"]
    seed = synth.STACK_SEED0
    x = synth.activations_bf16(cfg["seeds"][0], 1, H)
    lg = synth.router_logits(seed, 1, E)
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
    cfg = synth.WORKLOADS[args.workload]
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
        "config": {"workload": args.workload, "E": cfg["E"], "H": cfg["H"], "I": cfg["I"], "top_k": cfg["top_k"],
                   "T": 1, "layers": 1, "parallelism": "cpu oracle, 1 thread"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------------------------

def build_stack(cfg, layers, device):
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
        m = fe.MoELayer(E, H, I, max_T=cfg["T"], max_top_k=k)
        m.load_packed(gc, gs, dc, ds)
        handles.append(m)
    torch.cuda.synchronize()
    del Wgu, Wdn, gc, gs, dc, ds
    torch.cuda.empty_cache()
    return handles


def run_gpu(args):
    import torch

    import synth
    world, rank, local = dist_setup()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    workload = args.workload
    cfg = synth.WORKLOADS[workload]
    E, H, I, k, T = cfg["E"], cfg["H"], cfg["I"], cfg["top_k"], cfg["T"]
    layers = args.layers

    t_setup = time.perf_counter()
    stack = build_stack(cfg, layers, device)
    setup_s = time.perf_counter() - t_setup

    # inputs: x of layer 0, logits of every layer (seed 1000 + l); buffers reused by every replay
    x0_host = synth.activations_bf16(cfg["seeds"][0], T, H)
    lg_host = np.stack([synth.router_logits(synth.STACK_SEED0 + l, T, E, cfg["zipf"]) for l in range(layers)])
    x_pin = torch.from_numpy(x0_host.view(np.int16)).pin_memory()
    lg_pin = torch.from_numpy(lg_host).pin_memory()
    x_dev = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    lg_dev = torch.empty((layers, T, E), dtype=torch.float32, device=device)
    acts = [torch.empty((T, H), dtype=torch.bfloat16, device=device) for _ in range(layers)]
    y_pin = torch.empty((T, H), dtype=torch.int16).pin_memory()
    x_dev.copy_(x_pin.view(torch.bfloat16))
    lg_dev.copy_(lg_pin)

    s = torch.cuda.Stream(device=device)
    distinct = []

    def forward_all(stream):
        inp = x_dev
        for l, m in enumerate(stack):
            m.forward(inp, lg_dev[l], k, acts[l], stream=stream)
            inp = acts[l]

    with torch.cuda.stream(s):
        forward_all(s)
    torch.cuda.synchronize()
    # routing check of the stack: distinct experts per layer (for the byte count)
    for l, m in enumerate(stack):
        idx, _, _, _ = m.routing(T, k)
        distinct.append(len(set(idx.cpu().numpy().reshape(-1).tolist())))
    path, kernels_per_layer = stack[0].last_forward_info()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        forward_all(s)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    cur = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")   # lets a profiler select the timed launches
    e0.record(cur)
    for _ in range(args.steps):
        g.replay()
    e1.record(cur)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # keep the GPU busy while the sampler catches the clocks of a loaded GPU
    t_extra = time.perf_counter()
    while time.perf_counter() - t_extra < 0.5:
        for _ in range(20):
            g.replay()
        torch.cuda.synchronize()
    clk = clocks.stop()
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local, world, device)
    tokens_per_step_local = layers * T
    tokens_per_step = sum_over_ranks(tokens_per_step_local, world, device)
    value = tokens_per_step / (ms / 1e3)
    us_per_layer = ms * 1e3 / layers

    # end to end: pinned H2D of x and all logits, graph replay, D2H of the last layer's y
    h2d = x_pin.numel() * 2 + lg_pin.numel() * 4
    d2h = y_pin.numel() * 2
    for _ in range(3):
        x_dev.copy_(x_pin.view(torch.bfloat16), non_blocking=True)
        lg_dev.copy_(lg_pin, non_blocking=True)
        g.replay()
        y_pin.copy_(acts[-1].view(torch.int16), non_blocking=True)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0.record(cur)
    for _ in range(args.steps):
        x_dev.copy_(x_pin.view(torch.bfloat16), non_blocking=True)
        lg_dev.copy_(lg_pin, non_blocking=True)
        g.replay()
        y_pin.copy_(acts[-1].view(torch.int16), non_blocking=True)
    e1.record(cur)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, device)
    e2e_value = tokens_per_step / (e2e_ms / 1e3)

    peak, peak_kind = measured_peaks()
    bytes_layer = [algorithmic_bytes_per_layer(E, H, I, T, d) for d in distinct]
    bytes_step = float(sum(bytes_layer))
    achieved = bytes_step / (ms_local / 1e3) / 1e9
    prefill = workload.startswith("prefill")
    if prefill:
        # a dense contraction: FLOPs of gate_up + down over all token-expert pairs
        flops_layer = 2.0 * T * k * 3 * H * I
        tf = flops_layer * layers / (ms_local / 1e3) / 1e12
        tpeak, tpeak_kind = measured_tensor_peak()
        roofline = {"bound": "tensor", "achieved": tf, "peak": tpeak, "unit": "TFLOP/s", "frac": tf / tpeak,
                    "traffic": TRAFFIC.get(workload, (None,))[0], "kernel": KERNEL_NAMES.get(path, str(path)), "peak_kind": tpeak_kind,
                    "algorithmic_flops_per_layer": flops_layer,
                    "frac_of_nominal_fp4_9pflops": tf / 9000.0}
    else:
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "traffic": TRAFFIC.get(workload, (None,))[0], "kernel": KERNEL_NAMES.get(path, str(path)),
                    "peak_kind": peak_kind, "algorithmic_bytes_per_layer": bytes_layer[0]}
    if workload in TRAFFIC:
        roofline["traffic_kernel"] = TRAFFIC[workload][1]
        roofline["traffic_source"] = TRAFFIC[workload][2]
    line = {
        "metric": PREFILL_METRIC if prefill else METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded counter-based generator; random-init weights quantised to E2M1)",
        "config": {"workload": workload, "E": E, "H": H, "I": I, "top_k": k, "T": T, "layers_per_step": layers,
                   "global_batch": T * world, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: each step streams {layers} layers' routed experts "
                         f"({bytes_step / 1e9:.2f} GB)" if bytes_step > L2_BYTES else
                         f"step bytes ({bytes_step / 1e6:.0f} MB) fit in L2: not a valid HBM measurement",
                   "graph": f"one CUDA graph of {layers} chained fe_moe_forward calls"},
        "us_per_layer": us_per_layer,
        "hbm_gbs_achieved": achieved,
        "hbm_frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
        "roofline": roofline,
        "clocks": clk,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "gpu_launches": kernels_per_layer * layers * args.steps,
        "setup_s": setup_s,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        reps = args.cpu_reps
        per = time_oracle(cfg, reps)
        line["cpu_baseline"] = {"value": 1.0 / per, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"layer 0 of the stack, token 0, {reps} single-threaded oracle forwards"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fe", "reference"], default="fe")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--cpu-reps", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["decode_e128_t1", "decode_e128_t64_zipf", "decode_e512_t1", "decode_e512_t4",
                             "prefill_e128_t4096"])
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
