#!/usr/bin/env python3
"""Benchmark of the B200 Strata MoE layer: MoE-layer tokens/s and % roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl own|reference]
                    [--workload NAME] [--layers L]

A step is one forward of the whole layer (router -> top-k -> dispatch ->
quantised SwiGLU experts -> combine) over one batch of T tokens.  Steps rotate
over L independently seeded layers whose expert weights (L x 786 MB) exceed
the 126 MB L2, so no step finds its weights in L2 ("inputs larger than L2").
Each layer's forward is captured once in a CUDA graph and replayed.

Multi-GPU (torchrun): each rank runs its own replica on its own tokens (the
layer is token-parallel, so there is no data-path collective); `value` is the
tokens of all ranks over the max-over-ranks device time (weak scaling).

Prints ONE JSON line (rank 0).  `--impl reference` times the CPU oracle (the
plain C implementation the parity tests check against) on the host cores on
a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

WORKLOADS = {
    # name: (shape, T, description)
    "decode-t4": (gen.FLASH2, 4, "Flash-Next-shaped MoE layer, decode T=4 (MTP verify batch), "
                                 "2-bit block-32"),
    "decode-t1": (gen.FLASH2, 1, "Flash-Next-shaped MoE layer, decode T=1, 2-bit block-32"),
    "decode3-t64": (gen.FLASH3, 64, "Flash-Next-shaped MoE layer, batched decode T=64, "
                                    "3-bit block-32"),
    "prefill-t8192": (gen.FLASH2, 8192, "Flash-Next-shaped MoE layer, prefill chunk T=8192, "
                                        "2-bit block-32"),
    "tiny-t8": (gen.TINY, 8, "tiny MoE layer H256 E16 k2 I64, T=8"),
    "pruned256-t4": (gen.PRUNED256, 4, "pruned 256-expert build of the Flash-Next-shaped layer, "
                                       "decode T=4, 2-bit block-32"),
    "coder1-t4": (gen.CODER1, 4, "pruned 256-expert Coder build of the Flash-Next-shaped layer, "
                                 "decode T=4, 1-bit block-32"),
    "coder1-t8192": (gen.CODER1, 8192, "pruned 256-expert Coder build of the Flash-Next-shaped "
                                       "layer, prefill chunk T=8192, 1-bit block-32"),
    # 48-layer expert stack: h <- h + MoE(RMSNorm(h)) through 48 resident layers
    "stack48-t4": (gen.FLASH2, 4, "48-layer Flash-Next-shaped expert stack (~37 GB of 2-bit "
                                  "experts resident), decode T=4"),
    "stack48-t8192": (gen.FLASH2, 8192, "48-layer Flash-Next-shaped expert stack (~37 GB of "
                                        "2-bit experts resident), prefill chunk T=8192"),
}
STACK_LAYERS = 48
DEFAULT_WORKLOAD = "decode-t4"
STAGES = ["router", "topk", "dispatch", "gateup", "down", "combine"]
TIMING_NOTE = ("CUDA events recorded by the library on the launching stream around the kernel, "
               "in a second pass of the same graphs and workload right after the timed region")
GATEUP = 3


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index, period=0.005):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as ex:  # no NVML: report nothing rather than guess
            self.err = str(ex)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ helpers
def reduce_max(value: float, dist, device) -> float:
    """Max of `value` over all ranks (identity without a process group)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max / 1000.0)


def expert_bytes(shape):
    return shape.expert_bytes


def mat_bytes(shape):
    return shape.mat_code_bytes + 2 * shape.mat_scales


def traffic_from_profile(workload):
    """DRAM bytes per launch of the gate/up kernel from the committed ncu
    summary, or None when the summary is missing or was taken on an older
    version of the kernel source."""
    p = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    src = os.path.join(ROOT, d.get("source", ""))
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if h != d.get("source_sha256"):
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ CPU oracle
def oracle_throughput(layers, xs, shape, budget_s, threads):
    """Tokens/s of the CPU oracle over (layer, token) jobs, bounded by budget_s."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    jobs = [(l, t) for t in range(xs[0].shape[0]) for l in range(len(layers))]
    done = [0]
    lock = threading.Lock()
    t0 = time.perf_counter()

    def work(j):
        l, t = j
        if time.perf_counter() - t0 > budget_s:
            return
        oracle.moe_forward(layers[l], xs[l], sel=np.array([t], dtype=np.int32))
        with lock:
            done[0] += 1

    oracle.lib()
    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, jobs))
    dt = time.perf_counter() - t0
    return done[0] / dt, done[0], dt


def run_reference(args, wl):
    """The reference arm: the CPU oracle on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    shape, T, desc = WORKLOADS[wl]
    stack = wl.startswith("stack")  # a stack step passes every token through 48 layers
    n_layers = min(args.layers, 4)
    layers = [gen.layer_weights(shape, seed=0, layer=l) for l in range(n_layers)]
    xs = [gen.hidden(T, shape.hidden, seed=100, layer=l) for l in range(n_layers)]
    cores = os.cpu_count() or 1
    import oracle
    oracle.lib()
    # warm-up: W steps, each one token through one layer (untimed; bounded)
    budget = args.ref_budget
    tw = time.perf_counter()
    for i in range(min(args.warmup, 1)):
        oracle.moe_forward(layers[0], xs[0], sel=np.array([0], dtype=np.int32))
    del tw
    # timed: up to K steps of one token through one layer, all host cores
    from concurrent.futures import ThreadPoolExecutor
    done = [0]
    lock = threading.Lock()
    t0 = time.perf_counter()

    def step(i):
        if time.perf_counter() - t0 > budget:
            return
        l = i % n_layers
        t = (i // n_layers) % T
        oracle.moe_forward(layers[l], xs[l], sel=np.array([t], dtype=np.int32))
        with lock:
            done[0] += 1

    t0 = time.perf_counter()
    with ThreadPoolExecutor(cores) as ex:
        list(ex.map(step, range(args.steps)))
    dt = time.perf_counter() - t0
    value = done[0] / dt / (STACK_LAYERS if stack else 1)
    line = {
        "impl": "reference", "metric": "48-layer-stack tokens/s" if stack else "MoE-layer tokens/s",
        "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": done[0], "steps_requested": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1000 / max(done[0], 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl, "description": desc, "tokens_per_batch": T,
                   "layers_rotated": n_layers},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{done[0]} steps of one token through one layer (routing + "
                                   f"11 experts) across {n_layers} layers, {dt:.1f} s wall"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ own arm
def run_own(args, wl, emit=True, extra=None):
    """Time workload `wl`; print its JSON line (rank 0) when `emit`, and
    return it.  `extra` is merged into the line."""
    import torch
    import quantized_expert_ffn_04_b200 as qe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        if not dist.is_initialized():
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(local)
    dev = torch.cuda.current_device()
    shape, T, desc = WORKLOADS[wl]
    NL = args.layers
    peaks, peak_kind = load_peaks()

    # ---- layers (same weights on every rank, different tokens per rank)
    host_layers = []
    layers = []
    for l in range(NL):
        hw = gen.layer_weights(shape, seed=0, layer=l)
        layers.append(qe.Layer(hw, max_tokens=T, device=dev))
        if l < 2:
            host_layers.append(hw)
    xs_host = [gen.hidden(T, shape.hidden, seed=100 + rank, layer=l) for l in range(NL)]
    xs = [torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).cuda() for x in xs_host]
    ys = [torch.empty_like(x) for x in xs]
    stream = torch.cuda.current_stream()

    # ---- routing statistics for the algorithmic bytes (from the GPU's routing)
    distinct = []
    for l in range(NL):
        idx, _, _, _ = layers[l].route(xs[l])
        distinct.append(int(torch.unique(idx).numel()))
    torch.cuda.synchronize()

    # ---- probes: one CUDA event pair per (layer, stage), recorded by the library
    # on the launching stream around each stage.  They are captured into a
    # second set of graphs used only for the per-stage pass: event nodes between
    # kernels would also cut the programmatic-launch chain of the headline steps.
    decode = T <= 64
    # the fused decode layer is one kernel: its probe is the gate/up stage
    fused = decode and qe.strata_moe_launch_count(layers[0].handle, T) == 1
    stages = [GATEUP] if fused else ([0, 1] if T <= 256 else [0, 2]) + [3, 4, 5]
    ev_b = [[torch.cuda.Event(enable_timing=True) for _ in STAGES] for _ in range(NL)]
    ev_e = [[torch.cuda.Event(enable_timing=True) for _ in STAGES] for _ in range(NL)]
    for l in range(NL):
        for st in stages:
            ev_b[l][st].record(stream)
            ev_e[l][st].record(stream)
    torch.cuda.synchronize()

    def set_probes(on: bool):
        for l in range(NL):
            for st in stages:
                qe.strata_moe_set_probe(layers[l].handle, st,
                                        ev_b[l][st].cuda_event if on else None,
                                        ev_e[l][st].cuda_event if on else None)

    # ---- warm-up eagerly, then capture one graph per layer (plain and probed)
    for l in range(NL):
        layers[l].forward(xs[l], out=ys[l], stream=stream)
    torch.cuda.synchronize()
    for l in range(NL):
        layers[l].sync_status(stream)
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)

    def capture():
        gs = []
        for l in range(NL):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                layers[l].forward(xs[l], out=ys[l], stream=cap)
            gs.append(g)
        return gs

    graphs = capture()
    set_probes(True)
    graphs_probe = capture()
    set_probes(False)
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    for i in range(args.warmup):
        graphs[i % NL].replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()

    # ---- timed region: exactly K steps
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clocks:
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(args.steps):
            graphs[i % NL].replay()
        t_end.record(stream)
        torch.cuda.synchronize()
    ms = t_start.elapsed_time(t_end)
    for l in range(NL):
        layers[l].sync_status(stream)
    ms = reduce_max(ms, dist, "cuda")
    ms_step = ms / args.steps
    value = weak_scaling_value(T * args.steps, world, ms)

    # ---- per-stage pass: the probed graphs, same workload; each layer's event
    # pairs hold its last launch
    probe_steps = max(NL, min(args.steps, 200))
    for i in range(probe_steps):
        graphs_probe[i % NL].replay()
    torch.cuda.synchronize()
    for l in range(NL):
        layers[l].sync_status(stream)
    ran = list(range(NL))
    stage_ms = {STAGES[st]: statistics.mean(ev_b[l][st].elapsed_time(ev_e[l][st]) for l in ran)
                for st in stages}
    if fused:
        stage_ms["router+topk+dispatch+gateup+down+combine (fused)"] = stage_ms.pop("gateup")
    elif T <= 256:
        stage_ms["topk+dispatch"] = stage_ms.pop("topk")

    # ---- roofline of the dominant kernel (gate/up + SwiGLU)
    gu_ms = statistics.mean(ev_b[l][GATEUP].elapsed_time(ev_e[l][GATEUP]) for l in ran)
    if decode and fused:
        # the whole layer: router weight and bias, the distinct experts' packed
        # weights (all three matrices) and the shared expert's, token rows in and out
        gu_work = statistics.mean(shape.n_experts * shape.hidden * 4 + shape.n_experts * 4
                                  + (distinct[l] + 1) * shape.expert_bytes
                                  + 2 * T * shape.hidden * 2 for l in ran)
        achieved = gu_work / (gu_ms / 1000.0) / 1e9  # GB/s
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "kernel": "fused_decode_kernel (router, top-k, dispatch, gate/up, "
                "down, combine)", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": peak_kind + " hbm copy",
                "traffic": traffic_from_profile(wl), "algorithmic_bytes_per_launch": gu_work,
                "launch_ms": gu_ms, "timing": TIMING_NOTE}
    elif decode:
        mb = mat_bytes(shape)
        gu_work = statistics.mean((distinct[l] + 1) * 2 * mb + T * shape.hidden * 2 for l in ran)
        achieved = gu_work / (gu_ms / 1000.0) / 1e9  # GB/s
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "kernel": "gemv_gateup", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind + " hbm copy",
                "traffic": traffic_from_profile(wl), "algorithmic_bytes_per_launch": gu_work,
                "launch_ms": gu_ms, "timing": TIMING_NOTE}
    else:
        pairs = T * (shape.top_k + 1)
        ip = (shape.inter + 127) // 128 * 128
        gu_work = 2.0 * 2 * shape.hidden * ip * pairs  # gate + up, 2 flops per MAC
        achieved = gu_work / (gu_ms / 1000.0) / 1e12  # TFLOP/s
        # the gate/up launch is timed inside a ~2 ms layer step, not a
        # seconds-long loop: the burst peak applies
        peak = float(peaks["bf16_tflops"])
        roof = {"bound": "tensor", "kernel": "umma_expert_kernel (gate/up, fp16 operands)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_kind": peak_kind + " bf16 burst (fp16 runs at the bf16 rate)",
                "traffic": traffic_from_profile(wl), "algorithmic_flops_per_launch": gu_work,
                "launch_ms": gu_ms, "timing": TIMING_NOTE}
    step_bytes = [shape.n_experts * shape.hidden * 4 + shape.n_experts * 4
                  + (distinct[l] + 1) * shape.expert_bytes + 2 * T * shape.hidden * 2
                  for l in range(NL)]
    step_flops = 2.0 * 3 * shape.hidden * shape.inter * T * (shape.top_k + 1)

    # ---- e2e through the host-buffer entry point (pinned host memory)
    xh = [torch.from_numpy(x.view(np.int16).copy()).pin_memory() for x in xs_host]
    yh = [torch.empty_like(x).pin_memory() for x in xh]
    e2e_steps = min(args.steps, args.e2e_steps)
    for i in range(min(args.warmup, 8)):
        qe.strata_moe_forward_host(layers[i % NL].handle, xh[i % NL].data_ptr(), T,
                                   yh[i % NL].data_ptr(), stream.cuda_stream)
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(e2e_steps):
        l = i % NL
        qe.strata_moe_forward_host(layers[l].handle, xh[l].data_ptr(), T, yh[l].data_ptr(),
                                   stream.cuda_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1), dist, "cuda")
    e2e_value = weak_scaling_value(T * e2e_steps, world, e2e_ms)

    # ---- CPU baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cores = os.cpu_count() or 1
        v, n, dt = oracle_throughput(host_layers, xs_host[:len(host_layers)], shape,
                                     args.cpu_budget, cores)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} (layer, token) forwards of the same workload (routing + "
                         f"11 experts each) over {len(host_layers)} layers in {dt:.1f} s"}

    launches = qe.strata_moe_launch_count(layers[0].handle, T) * args.steps
    clk = clocks.summary()
    line = {
        "metric": "MoE-layer tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": wl, "description": desc, "tokens_per_batch": T,
                   "hidden": shape.hidden, "experts": shape.n_experts, "top_k": shape.top_k,
                   "inter": shape.inter, "bits": shape.bits, "layers_rotated": NL,
                   "l2": "inputs larger than L2: steps rotate over %d layers (%.1f GB of "
                         "expert weights)" % (NL, NL * (shape.n_experts + 1)
                                              * shape.expert_bytes / 1e9),
                   "cuda_graphs": True, "parallelism": f"replicas x{world}",
                   "arithmetic": "fp16 tensor-core operands with fp32 accumulation (decode: exact "
                                 "small-integer weights x fp16 tokens; prefill: fp16 dequantised "
                                 "weights), fp32 router, bf16 input and output"},
        "roofline": roof,
        "stages_ms": stage_ms,
        "step_bytes": statistics.mean(step_bytes),
        "step_hbm_frac": statistics.mean(step_bytes) / (ms_step / 1000.0) / 1e9
                         / float(peaks["hbm_gbs"]),
        "step_tflops": step_flops / (ms_step / 1000.0) / 1e12,
        "distinct_experts": statistics.mean(distinct),
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": T * shape.hidden * 2,
                "d2h_bytes_per_step": T * shape.hidden * 2, "steps": e2e_steps},
        "gpu_launches": launches,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                   "reasons": clk["reasons"], "samples": clk["samples"]},
    }
    if extra:
        line.update(extra)
    graphs.clear()
    graphs_probe.clear()
    for L in layers:
        L.close()
    if rank == 0 and emit:
        print(json.dumps(line), flush=True)
    if dist and emit:
        dist.barrier()
        dist.destroy_process_group()
    return line


# Workloads measured briefly after the default one (one GPU only), so the
# default line also carries the other decode shapes and the prefill:
# (workload, timed steps, layers rotated)
ALSO = [("decode-t1", 400, 8), ("decode3-t64", 100, 8), ("pruned256-t4", 400, 8),
        ("coder1-t4", 400, 8), ("prefill-t8192", 20, 4), ("coder1-t8192", 20, 4)]


def run_also(args):
    """Short runs of the ALSO workloads: value, step time and the dominant
    kernel's roofline per workload (no e2e or CPU leg).  A failing workload
    records its error instead of a number."""
    out = {}
    for wl, steps, nl in ALSO:
        a = argparse.Namespace(**vars(args))
        a.steps, a.warmup, a.layers, a.e2e_steps, a.no_cpu = steps, 3, nl, 1, True
        try:
            ln = run_own(a, wl, emit=False)
            r = ln["roofline"]
            out[wl] = {"value": ln["value"], "ms_per_step": ln["ms_per_step"], "steps": steps,
                       "layers_rotated": nl, "kernel_ms": r["launch_ms"],
                       "roofline_frac": r["frac"], "roofline_unit": r["unit"],
                       "roofline_peak": r["peak"], "clocks": ln["clocks"]}
        except Exception as e:  # noqa: BLE001 - recorded, the main line still prints
            out[wl] = {"error": f"{type(e).__name__}: {e}"[:300]}
    return out


def run_stack(args, wl):
    """One step = one pass of T tokens through the 48-layer stack
    (strata_moe_stack_forward: RMSNorm, MoE layer, residual, per layer), each
    step a CUDA graph that first restores the stack input."""
    import torch
    import quantized_expert_ffn_04_b200 as qe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    else:
        torch.cuda.set_device(local)
    dev = torch.cuda.current_device()
    shape, T, desc = WORKLOADS[wl]
    NL = STACK_LAYERS
    peaks, peak_kind = load_peaks()
    # layer 0's workspace serves the whole stack; the others need only their weights
    layers, host_layers = [], []
    for l in range(NL):
        hw = gen.layer_weights(shape, seed=0, layer=l)
        layers.append(qe.Layer(hw, max_tokens=T if l == 0 else 8, device=dev))
        if l < 2:
            host_layers.append(hw)
        del hw
    handles = [L.handle for L in layers]
    x0 = gen.hidden(T, shape.hidden, seed=200 + rank)
    h0 = torch.from_numpy(x0.view(np.int16).copy()).view(torch.bfloat16).cuda()
    h = torch.empty_like(h0)
    trace = torch.empty((NL, T, shape.hidden), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    # distinct experts per layer on the stack's own inputs (for the step bytes)
    h.copy_(h0)
    qe.strata_moe_stack_forward(handles, h.data_ptr(), T, trace.data_ptr(), stream.cuda_stream)
    layers[0].sync_status(stream)
    distinct = []
    if T <= 8:
        xn = torch.empty_like(h0)
        for l in range(NL):
            # the layer routes RMSNorm of its input
            qe.strata_moe_rmsnorm(trace[l].data_ptr(), xn.data_ptr(), T, shape.hidden,
                                  stream.cuda_stream)
            idx, _, _, _ = layers[l].route(xn)
            distinct.append(int(torch.unique(idx).numel()))
    torch.cuda.synchronize()

    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        h.copy_(h0)
        qe.strata_moe_stack_forward(handles, h.data_ptr(), T, None, cap.cuda_stream)
    stream.wait_stream(cap)
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    layers[0].sync_status(stream)
    if dist:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clocks:
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            g.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    layers[0].sync_status(stream)
    ms = reduce_max(t0.elapsed_time(t1), dist, "cuda")
    ms_step = ms / args.steps
    value = weak_scaling_value(T * args.steps, world, ms)

    # e2e: host buffers in and out around each pass (pinned)
    hh = torch.from_numpy(x0.view(np.int16).copy()).pin_memory()
    ho = torch.empty_like(hh).pin_memory()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        h.view(torch.int16).copy_(hh, non_blocking=True)
        qe.strata_moe_stack_forward(handles, h.data_ptr(), T, None, stream.cuda_stream)
        ho.copy_(h.view(torch.int16), non_blocking=True)
        stream.synchronize()
    e1.record(stream)
    torch.cuda.synchronize()
    layers[0].sync_status(stream)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dist, "cuda")
    e2e_value = weak_scaling_value(T * e2e_steps, world, e2e_ms)

    decode = T <= 64
    if decode:
        step_bytes = sum((d + 1) * shape.expert_bytes + shape.n_experts * shape.hidden * 4
                         for d in distinct)
        achieved = step_bytes / (ms_step / 1000.0) / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "kernel": "whole 48-layer step (router + fused decode kernel "
                "+ RMSNorm per layer)", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": peak_kind + " hbm copy", "traffic": None,
                "algorithmic_bytes_per_launch": step_bytes,
                "launch_ms": ms_step, "timing": "CUDA events around the timed graph replays"}
    else:
        ip = (shape.inter + 127) // 128 * 128
        flops = NL * 2.0 * 3 * shape.hidden * ip * T * (shape.top_k + 1)
        achieved = flops / (ms_step / 1000.0) / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
        roof = {"bound": "tensor", "kernel": "whole 48-layer step (expert GEMMs, router, "
                "dispatch, combine, RMSNorm per layer)", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_kind": peak_kind + " bf16 sustained (fp16 runs at the bf16 rate)",
                "traffic": None, "algorithmic_flops_per_launch": flops,
                "launch_ms": ms_step, "timing": "CUDA events around the timed graph replays"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cores = os.cpu_count() or 1
        xs_host = [gen.hidden(T, shape.hidden, seed=200, layer=l) for l in range(2)]
        v, n, dt = oracle_throughput(host_layers, xs_host, shape, args.cpu_budget, cores)
        cpu = {"value": v / NL, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} (layer, token) forwards (routing + 11 experts each) over 2 "
                         f"layers in {dt:.1f} s, divided by {NL} layers per stack pass"}
    clk = clocks.summary()
    per_layer = qe.strata_moe_launch_count(handles[0], T) + 1  # + RMSNorm
    line = {
        "metric": "48-layer-stack tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": wl, "description": desc, "tokens_per_batch": T,
                   "hidden": shape.hidden, "experts": shape.n_experts, "top_k": shape.top_k,
                   "inter": shape.inter, "bits": shape.bits, "layers": NL,
                   "l2": "inputs larger than L2: each step reads the experts of 48 layers "
                         "(%.1f GB resident)" % (NL * (shape.n_experts + 1)
                                                 * shape.expert_bytes / 1e9),
                   "cuda_graphs": True, "parallelism": f"replicas x{world}",
                   "arithmetic": "fp16 tensor-core operands with fp32 accumulation, fp32 "
                                 "router and RMSNorm, bf16 residual stream"},
        "roofline": roof,
        "distinct_experts": statistics.mean(distinct) if distinct else None,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": T * shape.hidden * 2,
                "d2h_bytes_per_step": T * shape.hidden * 2, "steps": e2e_steps},
        "gpu_launches": per_layer * NL * args.steps,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"],
                   "reasons": clk["reasons"], "samples": clk["samples"]},
    }
    del g
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--e2e-steps", type=int, default=1000)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=90.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-also", action="store_true",
                    help="skip the short runs of the other workloads that the default "
                         "workload's line carries")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args, args.workload)
    elif args.workload.startswith("stack"):
        run_stack(args, args.workload)
    elif (args.workload == DEFAULT_WORKLOAD and not args.no_also and args.gpus == 1
            and int(os.environ.get("WORLD_SIZE", "1")) == 1):
        # the headline first; the short runs after it can only add to its line
        line = run_own(args, args.workload, emit=False)
        line["other_workloads"] = run_also(args)
        print(json.dumps(line), flush=True)
    else:
        run_own(args, args.workload)


if __name__ == "__main__":
    main()
