#!/usr/bin/env python
"""Benchmark of the DeepSeek-V3 MoE layer forward pass on B200.

One step = one moe_forward (router, group-limited top-8 selection, permutation,
256 routed SwiGLU experts + the shared expert, weighted combine) over one
batch of T tokens whose inputs are already resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|skewed|fp8|tiny]
                    [--op layer|block|dense]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

`value` times the step alone (CUDA-graph replay, or eager steps with an L2 flush
for inputs that fit in L2); `e2e` times it with host buffers, the copy of x in
and of y out inside every step, through the C ABI's host-buffer entry point:
`e2e.value` with the steps alternating between two streams (one step's copies
overlap the other's kernels), `e2e.serial_value` one step after another.

The default run (decode) adds, under "workloads", the metric's other
configurations measured by the same code in the same process: prefill
(T=4096), skewed routing (T=16384) and FP8 weights (T=8192), 20 steps each
(--no-extra skips them).

With N > 1 (launched by torchrun) every rank runs an independent replica of
the layer on its own GPU and batch (weak scaling; the layer has no exchange
step on one node without expert parallelism).  Rank 0 prints one JSON line.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/sec (T=128 decode, T=4096 prefill); % of HBM/tensor roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernel per launch, from one ncu capture of that kernel on the workload itself (one
# pass of the two counters), keyed by workload: (bytes, kernel source hash the capture
# was taken at, how the figure was obtained).  A figure is reported only while the
# kernel sources still hash to the recorded value.
NCU_TRAFFIC: dict = {
    "decode": (8_626_317_824, "dc7b90005eef3c61",
              "ncu capture of this workload's moe_gemm_kernel<0, 32> launch: "
              "dram__bytes_read.sum + dram__bytes_write.sum"),
    "prefill": (16_519_067_904, "dc7b90005eef3c61",
               "ncu capture of this workload's moe_gemm2_kernel<0> launch: "
               "dram__bytes_read.sum + dram__bytes_write.sum"),
    "skewed": (12_199_695_616, "dc7b90005eef3c61",
              "ncu capture of this workload's moe_gemm2_kernel<0> launch: "
              "dram__bytes_read.sum + dram__bytes_write.sum"),
    "fp8": (9_041_506_560, "dc7b90005eef3c61",
           "ncu capture of this workload's moe_gemm2_fp8_kernel<0> launch: "
           "dram__bytes_read.sum + dram__bytes_write.sum"),
}

HBM_NOMINAL_GBS = 7700.0  # B200 (HGX) HBM3e nominal bandwidth, for context beside the measured copy peak


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "fine_grained_moe_gemm_b200", "csrc")
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def time_e2e(e2e_step, steps: int, warmup: int, streams, device, barrier=lambda: None, flush=None):
    """End-to-end step times with host buffers, in ms over `steps` steps: (serial, pipelined).
    e2e_step(i, s) enqueues step i (copy in, layer, copy out) on stream s, alternating between
    two buffer sets by i % 2.  serial: one stream, per-step events summed (an L2 flush between
    steps when `flush` is given).  pipelined: steps alternate between the two streams, so one
    step's copies overlap the other's kernels; first copy to last copy.  None without a flush
    only (small inputs are measured serially)."""
    import torch

    def pipelined(n):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(streams[0])
        streams[1].wait_event(t0)
        for i in range(n):
            e2e_step(i, streams[i % 2])
        done = torch.cuda.Event()
        done.record(streams[1])
        streams[0].wait_event(done)
        t1.record(streams[0])
        return t0, t1

    for i in range(max(warmup, 1)):
        e2e_step(i, streams[0])
    pipelined(2 * max(warmup, 1))
    torch.cuda.synchronize()
    barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xff)
        evs[i][0].record(streams[0])
        e2e_step(i, streams[0])
        evs[i][1].record(streams[0])
    torch.cuda.synchronize()
    serial = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), device)
    pipe = None
    if flush is None:
        barrier()
        p0, p1 = pipelined(steps)
        torch.cuda.synchronize()
        pipe = max_over_ranks(p0.elapsed_time(p1), device)
    return serial, pipe


def e2e_entry(tokens: float, serial_ms: float, pipe_ms, h2d: int, d2h: int, api: str) -> dict:
    best = pipe_ms if pipe_ms is not None else serial_ms
    return {"value": round(tokens / (best / 1e3), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "api": api, "mode": "pipelined" if pipe_ms is not None else "serial",
            "serial_value": round(tokens / (serial_ms / 1e3), 1),
            "pipeline": ("steps alternate between two streams and two buffer sets: one step's host copies "
                         "overlap the other step's kernels") if pipe_ms is not None else None}


def max_over_ranks(x: float, device) -> float:
    """The slowest rank's figure: every rank of the process group takes part (a no-op in
    a single process).  Timings are device-measured per rank, then reduced here."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {k: float(j[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            try:
                bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception:
            self._h = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                util = nv.nvmlDeviceGetUtilizationRates(self._h).gpu
                self.samples.append((mhz, r, util))
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if self._h is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": len(self.samples)}
        busy = [s for s in self.samples if s[2] > 0] or self.samples
        bits = 0
        for s in busy:
            bits |= s[1]
        names = [n for b, n in self.REASONS.items() if bits & b and b != 0x1]
        return {"sm_mhz": statistics.median(s[0] for s in busy), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(busy)}


# --------------------------------------------------------------------------- accounting
def layer_accounting(wl, T, U, out_bytes):
    """Algorithmic flops / bytes of one layer step: the weights of the U touched
    routed experts + the shared expert + the router, x read once, y written once."""
    wb = 1 if wl.fp8 else 2
    F = T * wl.flops_per_token
    B = ((U + 1) * 3 * wl.hidden * wl.d * wb + wl.n_experts * wl.d * 2 + T * wl.d * 2 + T * wl.d * out_bytes)
    if wl.fp8:
        B += (U + 1) * 3 * (wl.hidden // 128) * (wl.d // 128) * 4
    return F, B


def kernel_accounting(wl, T, U, stage):
    """Algorithmic flops / bytes of one launch of a grouped GEMM.
    gate_up: gate+up weights of the touched experts, the permuted x rows read
    once, h written once.  down: down weights, h read once, fp32 combine
    buffer written once."""
    wb = 1 if wl.fp8 else 2
    rows = T * wl.top_k + T
    if stage == "gate_up":
        F = rows * 2 * 2 * wl.hidden * wl.d
        B = (U + 1) * 2 * wl.hidden * wl.d * wb + rows * wl.d * 2 + rows * wl.hidden * 2
    else:
        F = rows * 2 * wl.hidden * wl.d
        B = (U + 1) * wl.hidden * wl.d * wb + rows * wl.hidden * 2 + T * wl.d * 4
    return F, B


FP8_OVER_BF16 = 2.0  # nominal dense e4m3 / bf16 tensor throughput ratio (4.5 / 2.25 PFLOP/s)


L2_BYTES = 126 * 2**20
SUSTAINED_AFTER_S = 0.1  # a tensor-bound run this long is timed under the power cap


def tensor_peak(peaks, fp8, sustained=False):
    """Measured bf16 tensor peak (TFLOP/s): the burst figure, or the one sustained under the
    power cap for kernels timed inside a long run; an e4m3 contraction takes it times the
    nominal ratio."""
    return peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"] * (FP8_OVER_BF16 if fp8 else 1.0)


def roofline(F, B, seconds, peaks, peak_kind, fp8=False, sustained=False):
    ptc = tensor_peak(peaks, fp8, sustained)
    t_tc = F / (ptc * 1e12)
    t_hbm = B / (peaks["hbm_gbs"] * 1e9)
    if t_hbm >= t_tc:
        ach = B / seconds / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 4),
                "peak_source": peak_kind + " copy bandwidth (read + write stream); a read-mostly kernel can exceed it",
                "frac_of_nominal": round(ach / HBM_NOMINAL_GBS, 4), "nominal_gbs": HBM_NOMINAL_GBS}
    ach = F / seconds / 1e12
    src = peak_kind + (" sustained" if sustained else " burst") + (" bf16 x 2 (nominal e4m3/bf16 ratio)" if fp8 else "")
    out = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(ptc, 1), "unit": "TFLOP/s",
           "frac": round(ach / ptc, 4), "peak_source": src}
    if sustained:
        out["frac_of_burst_peak"] = round(ach / tensor_peak(peaks, fp8), 4)
    return out


# --------------------------------------------------------------------------- oracle timing
def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_runner(wl, W, x, n_tokens, threads):
    """The CPU oracle alone (nothing of the CUDA path) on the batch.  Returns
    (route, experts, n): route() runs the router GEMM (fp64), the selection and the
    permutation on all T tokens; experts() runs the expert math and the combine on
    n sampled tokens, chosen among the first 512 to share experts (that keeps the
    host copy of the weights small; every token costs the same k routed + 1 shared
    expert evaluations, so the per-token cost does not depend on the choice)."""
    import numpy as np
    import torch

    import oracle

    T = x.shape[0]

    def u16(t):
        return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def u8(t):
        return t.detach().contiguous().view(torch.uint8).cpu().numpy()

    x_h = x.cpu().numpy() if x.dtype == torch.float32 else u16(x)
    wr_h = u16(W["w_router"])
    bias_h = W["bias"].cpu().numpy()
    pool = min(T, 512)
    idx_p, _ = oracle.select(oracle.router_logits(x_h[:pool], wr_h), bias_h, wl.n_groups, wl.topk_groups, wl.top_k)
    chosen, experts = [], set()
    while len(chosen) < min(n_tokens, pool):
        best = min((t for t in range(pool) if t not in chosen), key=lambda t: (len(set(idx_p[t]) - experts), t))
        chosen.append(best)
        experts |= set(idx_p[best].tolist())
    toks = np.array(sorted(chosen), dtype=np.int32)

    conv = u8 if wl.fp8 else u16
    E = wl.n_experts
    wg, wu, wd = [None] * E, [None] * E, [None] * E
    kw = {}
    if wl.fp8:
        sg, su, sd = [None] * E, [None] * E, [None] * E
    for e in sorted(experts):
        wg[e], wu[e], wd[e] = conv(W["w_gate"][e]), conv(W["w_up"][e]), conv(W["w_down"][e])
        if wl.fp8:
            sg[e], su[e], sd[e] = (W["s_gate"][e].cpu().numpy(), W["s_up"][e].cpu().numpy(),
                                   W["s_down"][e].cpu().numpy())
    if wl.fp8:
        kw = dict(s_gate=sg, s_up=su, s_down=sd, ss_gate=W["ss_gate"].cpu().numpy(),
                  ss_up=W["ss_up"].cpu().numpy(), ss_down=W["ss_down"].cpu().numpy())
    L = oracle.Layer(wl.d, E, wl.hidden, wl.shared_hidden, wl.top_k, wl.routed_scale, wg, wu, wd,
                     conv(W["ws_gate"]), conv(W["ws_up"]), conv(W["ws_down"]), x_is_f32=wl.x_f32, **kw)
    routing = {}

    def route():
        l = oracle.router_logits(x_h, wr_h)
        routing["idx"], routing["w"] = oracle.select(l, bias_h, wl.n_groups, wl.topk_groups, wl.top_k)
        oracle.permute(routing["idx"], wl.n_experts)

    def run_experts():
        oracle.expert_tokens(L, x_h, routing["idx"], routing["w"], toks, n_threads=threads)

    return route, run_experts, len(toks)


def oracle_step_time(wl, route, run_experts, n):
    """Seconds of one oracle step over the whole batch: routing and permutation of all
    T tokens as timed, plus the sampled expert math scaled to T by its per-token cost."""
    t0 = time.perf_counter()
    route()
    t1 = time.perf_counter()
    run_experts()
    t2 = time.perf_counter()
    return (t1 - t0) + (t2 - t1) * wl.T / n, t1 - t0, t2 - t1


def oracle_sample_desc(wl, n, threads):
    return (f"router GEMM (fp64), selection and permutation on all {wl.T} tokens; expert math and combine on "
            f"{n} of them (chosen to share experts) and scaled to {wl.T} by the per-token cost (every token costs "
            f"k routed + 1 shared expert evaluations); fp64; {threads} host threads")


def _cfg(wl):
    import fine_grained_moe_gemm_b200 as moe
    return moe.MoeConfig(wl.d, wl.n_experts, wl.n_groups, wl.topk_groups, wl.top_k, wl.hidden, 1, wl.shared_hidden,
                         wl.routed_scale, moe.MOE_F32 if wl.x_f32 else moe.MOE_BF16,
                         moe.MOE_E4M3 if wl.fp8 else moe.MOE_BF16)


def workload_desc(wl):
    w = (f"{wl.name}: DeepSeek-V3 MoE layer forward, T={wl.T}, d={wl.d}, {wl.n_experts} routed experts in "
         f"{wl.n_groups} groups (top-{wl.topk_groups} groups, top-{wl.top_k} experts), SwiGLU hidden {wl.hidden}, "
         f"1 shared expert (hidden {wl.shared_hidden}), routed scale {wl.routed_scale}")
    if wl.fp8:
        w += ", e4m3 expert weights with 128x128 fp32 block scales, activations e4m3 per 1x128"
    if wl.bias == "hot":
        w += f", selection bias +{wl.hot_bias} on {wl.n_hot} Zipf({wl.zipf_s}) hot experts"
    elif wl.bias == "zero":
        w += ", selection bias 0"
    else:
        w += ", selection bias U[-0.1, 0.1]"
    return w


# --------------------------------------------------------------------------- arms
def run_reference(args, wl):
    """The CPU oracle, as it stands, on the host cores: each step is the whole batch's
    routing plus a bounded sample of its expert math (see cpu_baseline.sample)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch

    from workloads import make_inputs
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if dev == "cpu" and wl.d > 1024:
        print(json.dumps({"impl": "reference", "unavailable": "full-size synthetic weights are generated on a GPU"}))
        return 0
    W = make_inputs(wl, dev)
    W = {k: v.to("cuda") for k, v in W.items()} if dev == "cuda" else W
    threads = host_cores()
    n = args.cpu_sample or min(wl.T, 2 * threads)
    route, run_experts, n = _oracle_runner(wl, W, W["x"], n, threads)
    for _ in range(args.warmup):
        oracle_step_time(wl, route, run_experts, n)
    total = 0.0
    for _ in range(args.steps):
        total += oracle_step_time(wl, route, run_experts, n)[0]
    value = wl.T * args.steps / total
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(wl), "T": wl.T},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": oracle_sample_desc(wl, n, threads)},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


class RunContext:
    """One process per GPU: device, ranks, the barrier and the peaks."""

    def __init__(self):
        import torch
        import torch.distributed as dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(self.local)
        self.dev = torch.device("cuda", self.local)
        if self.world > 1:
            import datetime
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=self.dev)
        self.peaks, self.peak_kind = load_peaks()

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def close(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


def measure_layer(args, wl, steps, warmup, ctx, block=False):
    """One workload of the layer (or of the pre-norm sublayer with block=True):
    device-only steps, stage times, the end-to-end steps with host buffers, and the
    accounting.  Every rank runs it (same collective steps in the same order);
    returns (entry, W, x) with the timings already reduced as the max over ranks."""
    import torch

    import fine_grained_moe_gemm_b200 as moe
    from workloads import make_inputs, make_norm_gain, make_stream

    dev, rank, world = ctx.dev, ctx.rank, ctx.world
    peaks, peak_kind = ctx.peaks, ctx.peak_kind
    cfg = _cfg(wl)
    T = wl.T
    src_dev = "cpu" if wl.d <= 1024 else dev
    W = {k: v.to(dev) for k, v in make_inputs(wl, src_dev, seed=rank).items()}
    weights = {k: v for k, v in W.items() if k not in ("x", "bias")}
    x, bias = W["x"], W["bias"]
    norm_g = None
    if block:  # the input is the residual stream h; the layer runs on RMSNorm(h) and adds h back
        x = W["x"] = make_stream(wl, dev, seed=rank)
        norm_g = W["norm_g"] = make_norm_gain(wl, dev, seed=rank)
    ws_size = moe.block_workspace_size(cfg, T) if block else moe.workspace_size(cfg, T)
    ws = torch.empty(ws_size, dtype=torch.uint8, device=dev)
    y = torch.empty((T, wl.d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def forward(xin, ev=None):
        if block:
            moe.moe_forward_block(cfg, weights, norm_g, xin, bias, y, workspace=ws, stage_events=ev)
        else:
            moe.moe_forward(cfg, weights, xin, bias, y, workspace=ws, stage_events=ev)

    # inputs smaller than twice the L2 would be served from it: write a buffer larger than
    # the L2 before every timed step and time the steps alone (events around each step)
    in_bytes = sum(v.numel() * v.element_size() for v in W.values())
    flush = torch.empty(4 * L2_BYTES, dtype=torch.uint8, device=dev) if in_bytes < 2 * L2_BYTES else None

    for _ in range(max(warmup, 0)):
        forward(x)
    torch.cuda.synchronize()
    if moe.device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    plan = moe.forward_plan(cfg, T)
    if block:
        plan["launches"] += 1  # the norm (with e4m3 weights it also writes the codes the copy then moves)
    graph = None
    # serving-style timing: the whole step captured once as a CUDA graph and replayed (no host launch
    # gaps); with an L2 flush between steps the steps are launched and timed one by one instead
    if not args.eager and flush is None:
        # stage times from eager steps (the graph runs the same kernels), then one captured step
        for i in range(steps):
            forward(x, evs[i])
        torch.cuda.synchronize()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        n0 = moe.launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            forward(x)
        if moe.launch_count() - n0 != plan["launches"]:
            raise RuntimeError("the captured step does not hold the planned kernels")
        graph.replay()
        torch.cuda.synchronize()
    ctx.barrier()
    torch.cuda.synchronize()
    n_launch0 = moe.launch_count()
    with ClockSampler(ctx.local) as clk:
        t_start.record(stream)
        for i in range(steps):
            if flush is not None:
                flush.fill_(i & 0xff)
            if graph is not None:
                graph.replay()
            else:
                forward(x, evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    # kernels that ran in the timed region: counted at launch, or the captured step's per replay
    launches = moe.launch_count() - n_launch0 if graph is None else plan["launches"] * steps
    if launches != plan["launches"] * steps:
        raise RuntimeError(f"{launches} kernel launches in the timed region, the plan says "
                           f"{plan['launches']} per step")
    ctx.barrier()
    ms = t_start.elapsed_time(t_end) if flush is None else sum(e[0].elapsed_time(e[5]) for e in evs)
    stage_ms = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
                for i, name in enumerate(moe.STAGES)}
    ms_max = max_over_ranks(ms, dev)
    if moe.device_error() != 0:
        raise RuntimeError("device error word set during the timed steps")
    used_graph, flushed = graph is not None, flush is not None
    del graph

    # end to end with host buffers: pinned x in, y out, every step.  The layer goes through
    # moe_forward_host (the C ABI call that takes host buffers and does the copies); the block,
    # which has no host entry point, copies around moe_forward_block.  Measured two ways:
    #   serial     one stream: copy in, layer, copy out, step after step (per-step events, summed)
    #   pipelined  steps alternate between two streams with two workspaces, so the copies of
    #              one step run on the copy engines while the other step's kernels run (the
    #              loop a server runs); timed from the first copy to the last one.
    e2e_steps = max(1, steps)
    x_host = x.cpu().pin_memory()
    y_hosts = [torch.empty((T, wl.d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    streams = [stream, torch.cuda.Stream()]
    if block:
        x_devs = [torch.empty_like(x) for _ in range(2)]
        y_devs = [y, torch.empty_like(y)]
        e2e_ws = [ws, torch.empty_like(ws)]
    else:
        hws = moe.host_workspace_size(cfg, T, torch.bfloat16)
        e2e_ws = [torch.empty(hws, dtype=torch.uint8, device=dev) for _ in range(2)]

    def e2e_step(i, s):
        j = i % 2
        if block:
            with torch.cuda.stream(s):
                x_devs[j].copy_(x_host, non_blocking=True)
                moe.moe_forward_block(cfg, weights, norm_g, x_devs[j], bias, y_devs[j], workspace=e2e_ws[j],
                                      stream=s)
                y_hosts[j].copy_(y_devs[j], non_blocking=True)
        else:
            moe.moe_forward_host(cfg, weights, x_host, bias, y_hosts[j], workspace=e2e_ws[j], stream=s)

    e2e_serial_ms, e2e_pipe_ms = time_e2e(e2e_step, e2e_steps, warmup, streams, dev, ctx.barrier, flush)
    if moe.device_error() != 0:
        raise RuntimeError("device error word set during the end-to-end steps")
    del e2e_ws, ws, flush

    # routed experts actually touched (for the byte accounting), through the ABI
    logits = torch.empty((T, wl.n_experts), dtype=torch.float32, device=dev)
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device=dev)
    wsel = torch.empty((T, wl.top_k), dtype=torch.float32, device=dev)
    xr = x
    if block:
        xr = torch.empty_like(x)
        moe.moe_rmsnorm(x, norm_g, xr)
    moe.moe_route(cfg, xr, W["w_router"], logits, bias, idx, wsel)
    counts = torch.empty(wl.n_experts, dtype=torch.int32, device=dev)
    offs = torch.empty(wl.n_experts + 1, dtype=torch.int32, device=dev)
    srcp = torch.empty(T * wl.top_k, dtype=torch.int32, device=dev)
    invp = torch.empty(T * wl.top_k, dtype=torch.int32, device=dev)
    moe.moe_permute(cfg, idx, counts, offs, srcp, invp)
    c = counts.cpu()
    U = int((c > 0).sum())

    F, B = layer_accounting(wl, T, U, 2)
    step_s = ms_max / steps / 1e3
    k_name = max(("gate_up", "down+combine"), key=lambda n: stage_ms[n])
    kF, kB = kernel_accounting(wl, T, U, "gate_up" if k_name == "gate_up" else "down")
    sus = ms_max / 1e3 >= SUSTAINED_AFTER_S
    kr = roofline(kF, kB, stage_ms[k_name] / 1e3, peaks, peak_kind, fp8=wl.fp8, sustained=sus)
    kr["kernel"] = ("moe_gemm2" if plan["cta_pair"] else "moe_gemm") + ("_fp8" if plan["fp8"] else "") + \
        "_kernel<" + ("GATEUP" if k_name == "gate_up" else "DOWN") + ", BN=" + str(plan["token_tile"]) + ">"
    tr = NCU_TRAFFIC.get(wl.name + (":block" if block else ""))
    ok = tr is not None and tr[1] == kernel_source_hash()
    kr["traffic"] = tr[0] if ok else None
    kr["traffic_source"] = tr[2] if ok else "none: no ncu capture of the current kernel sources for this workload"
    lr = roofline(F, B, step_s, peaks, peak_kind, fp8=wl.fp8, sustained=sus)
    # the router GEMM stays bf16 in the FP8 layer
    F_router = 2 * T * wl.n_experts * wl.d
    t_tc = ((F - F_router) / (tensor_peak(peaks, wl.fp8, sus) * 1e12)
            + F_router / (tensor_peak(peaks, False, sus) * 1e12))
    t_roof = max(t_tc, B / (peaks["hbm_gbs"] * 1e9))
    lr["roofline_ms"] = round(t_roof * 1e3, 4)
    lr["frac_of_roofline_time"] = round(t_roof / step_s, 4)
    lr["algorithmic_bytes"] = B
    lr["algorithmic_flops"] = F
    kr["algorithmic_bytes"] = kB
    kr["algorithmic_flops"] = kF
    value = world * T * steps / (ms_max / 1e3)
    entry = {
        "value": round(value, 1), "unit": UNIT, "steps": steps, "warmup": warmup,
        "ms_per_step": round(ms_max / steps, 4), "dtype": "e4m3" if wl.fp8 else "bf16",
        "config": {"workload": ("MoE sublayer y = h + MoE(RMSNorm(h)), eps 1e-6, bf16 residual stream; "
                                if block else "") + workload_desc(wl), "T": T, "experts_touched": U,
                   "max_rows_per_expert": int(c.max()), "mean_rows_per_touched_expert": round(T * wl.top_k / U, 1),
                   "l2": ("inputs larger than L2: the touched expert weights "
                          f"({(U + 1) * 3 * wl.hidden * wl.d * (1 if wl.fp8 else 2) / 1e9:.2f} GB) stream from HBM "
                          "every step") if not flushed else
                         ("L2 flushed before every timed step (a 504 MiB buffer written between steps, outside "
                          "the per-step CUDA events that are summed)"),
                   "parallelism": f"replicas x{world} (no data-path collective)",
                   "launch": "CUDA-graph replay of the captured step" if used_graph else "eager"},
        "roofline": kr,
        "layer_roofline": lr,
        "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "e2e": e2e_entry(world * T * e2e_steps, e2e_serial_ms, e2e_pipe_ms, x.numel() * x.element_size(),
                         y.numel() * y.element_size(),
                         "moe_forward_block + copies" if block else "moe_forward_host (host buffers)"),
        "gpu_launches": launches,
        "plan": plan,
        "clocks": clk.summary(),
    }
    return entry, W, x


EXTRA_WORKLOADS = ("prefill", "skewed", "fp8")
EXTRA_STEPS = 20


def run_ours(args, wl):
    import torch

    from workloads import WORKLOADS

    ctx = RunContext()
    block = args.op == "block"
    entry, W, x = measure_layer(args, wl, args.steps, args.warmup, ctx, block=block)
    cpu = None
    if ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline and not block:
        threads = host_cores()
        n = args.cpu_sample or min(wl.T, 2 * threads)
        route, run_experts, n = _oracle_runner(wl, W, x, n, threads)
        sec, t_route, t_exp = oracle_step_time(wl, route, run_experts, n)
        cpu = {"value": round(wl.T / sec, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": oracle_sample_desc(wl, n, threads),
               "seconds": {"routing_all_tokens": round(t_route, 3), "experts_sample": round(t_exp, 3)}}
    del W, x
    torch.cuda.empty_cache()
    # the metric's other configurations, measured by the same code in the same run
    subs = {}
    if not args.no_extra and not block and args.tokens == 0 and wl.name == "decode":
        for name in EXTRA_WORKLOADS:
            e, W2, x2 = measure_layer(args, WORKLOADS[name], min(args.steps, EXTRA_STEPS), args.warmup, ctx)
            del W2, x2
            torch.cuda.empty_cache()
            subs[name] = e
    ctx.close()
    if ctx.rank == 0:
        line = {"metric": METRIC, "value": entry["value"], "unit": UNIT, "n_gpus": ctx.world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": entry["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": entry["dtype"],
                "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights; no checkpoint)"}
        for k in ("config", "roofline", "layer_roofline", "stages_ms", "e2e", "gpu_launches", "plan", "clocks"):
            line[k] = entry[k]
        if subs:
            line["workloads"] = subs
        line["kernel_source"] = kernel_source_hash()
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line))
    return 0


def run_dense(args, wl):
    """The dense SwiGLU FFN of the model's first layers (d -> 18432 -> d) on the same
    grouped-GEMM kernels, at the workload's T (e4m3 weights for the FP8 workload)."""
    import torch
    import torch.distributed as dist

    import fine_grained_moe_gemm_b200 as moe
    from workloads import DENSE_HIDDEN, make_dense_weights, make_x

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peaks, peak_kind = load_peaks()
    T, d, Hd = wl.T, wl.d, DENSE_HIDDEN
    W = make_dense_weights(d, Hd, wl.fp8, dev, seed=rank)
    x = make_x(wl, dev, seed=rank)
    act = moe.MOE_BF16
    wdt = moe.MOE_E4M3 if wl.fp8 else moe.MOE_BF16
    ws = torch.empty(moe.dense_workspace_size(d, Hd, act, wdt, T), dtype=torch.uint8, device=dev)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def forward(xin, ev=None):
        moe.moe_dense_ffn(W["w_gate"], W["w_up"], W["w_down"], xin, y, W.get("s_gate"), W.get("s_up"),
                          W.get("s_down"), workspace=ws, stage_events=ev)

    for _ in range(max(args.warmup, 0)):
        forward(x)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # tables, two GEMMs and the cast; e4m3 adds the quantisation of x (fused with its copy into row order)
    per_step = 5 if wl.fp8 else 4
    for i in range(args.steps):  # stage times from eager steps, then the step captured once
        forward(x, evs[i])
    torch.cuda.synchronize()
    graph = None
    if not args.eager:
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        n0 = moe.launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            forward(x)
        if moe.launch_count() - n0 != per_step:
            raise RuntimeError("the captured dense step does not hold the planned kernels")
        graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = moe.launch_count()
    with ClockSampler(local) as clk:
        t0.record(stream)
        for i in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                forward(x)
        t1.record(stream)
        torch.cuda.synchronize()
    launches = moe.launch_count() - n0 if graph is None else per_step * args.steps
    if launches != per_step * args.steps or moe.device_error() != 0:
        raise RuntimeError(f"dense FFN: {launches} launches, device error word set or not as planned")
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    stage_ms = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, name in enumerate(moe.STAGES)}
    # end to end with host buffers (copies around moe_dense_ffn), serial and pipelined as for the layer
    x_host = x.cpu().pin_memory()
    y_hosts = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_devs, y_devs, wss = [torch.empty_like(x) for _ in range(2)], [y, torch.empty_like(y)], [ws, torch.empty_like(ws)]

    def e2e_step(i, s):
        j = i % 2
        with torch.cuda.stream(s):
            x_devs[j].copy_(x_host, non_blocking=True)
            moe.moe_dense_ffn(W["w_gate"], W["w_up"], W["w_down"], x_devs[j], y_devs[j], W.get("s_gate"),
                              W.get("s_up"), W.get("s_down"), workspace=wss[j], stream=s)
            y_hosts[j].copy_(y_devs[j], non_blocking=True)

    barrier = (lambda: dist.barrier()) if world > 1 else (lambda: None)
    e2e_serial_ms, e2e_pipe_ms = time_e2e(e2e_step, args.steps, args.warmup, [stream, torch.cuda.Stream()], dev,
                                          barrier)
    if moe.device_error() != 0:
        raise RuntimeError("dense FFN: device error word set during the end-to-end steps")
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    wb = 1 if wl.fp8 else 2
    sc = 3 * (d // 128) * (Hd // 128) * 4 if wl.fp8 else 0
    F = 2 * 3 * d * Hd * T
    B = 3 * d * Hd * wb + sc + 2 * T * d * 2
    sus = ms / 1e3 >= SUSTAINED_AFTER_S
    step_s = ms / args.steps / 1e3
    lr = roofline(F, B, step_s, peaks, peak_kind, fp8=wl.fp8, sustained=sus)
    t_roof = max(F / (tensor_peak(peaks, wl.fp8, sus) * 1e12), B / (peaks["hbm_gbs"] * 1e9))
    lr.update({"roofline_ms": round(t_roof * 1e3, 4), "frac_of_roofline_time": round(t_roof / step_s, 4),
               "algorithmic_bytes": B, "algorithmic_flops": F})
    k_name = max(("gate_up", "down+combine"), key=lambda n: stage_ms[n])
    if k_name == "gate_up":
        kF, kB = 2 * 2 * d * Hd * T, 2 * d * Hd * wb + 2 * sc // 3 + T * d * 2 + T * Hd * 2
    else:
        kF, kB = 2 * d * Hd * T, d * Hd * wb + sc // 3 + T * Hd * 2 + T * d * 4
    kr = roofline(kF, kB, stage_ms[k_name] / 1e3, peaks, peak_kind, fp8=wl.fp8, sustained=sus)
    kr.update({"kernel": k_name + " grouped GEMM (one group of T rows)", "traffic": None,
               "algorithmic_bytes": kB, "algorithmic_flops": kF})
    line = {
        "metric": METRIC, "value": round(world * T * args.steps / (ms / 1e3), 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if wl.fp8 else "bf16",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights; no checkpoint)",
        "config": {"workload": f"dense SwiGLU FFN d={d} -> {Hd} -> {d} (the model's first layers), T={T}"
                               + (", e4m3 weights with 128x128 fp32 block scales" if wl.fp8 else ""),
                   "T": T, "l2": f"inputs larger than L2: {3 * d * Hd * wb / 1e9:.2f} GB of weights stream every step",
                   "parallelism": f"replicas x{world} (no data-path collective)"},
        "roofline": kr, "layer_roofline": lr, "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "e2e": e2e_entry(world * T * args.steps, e2e_serial_ms, e2e_pipe_ms, x.numel() * x.element_size(),
                         y.numel() * y.element_size(), "moe_dense_ffn + copies"),
        "gpu_launches": launches, "clocks": clk.summary(), "kernel_source": kernel_source_hash(),
    }
    line["config"]["launch"] = "CUDA-graph replay of the captured step" if graph is not None else "eager"
    print(json.dumps(line))
    return 0


def main():
    from workloads import WORKLOADS

    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    p.add_argument("--cpu-sample", type=int, default=0,
                   help="tokens of the oracle's expert-math sample (0: min(T, 2 x host cores))")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="decode only: skip the prefill, skewed and fp8 lines added under 'workloads'")
    p.add_argument("--tokens", type=int, default=0, help="override the workload's T (sweeps; default: as named)")
    p.add_argument("--eager", action="store_true",
                   help="launch every timed step from the host instead of replaying the captured step as a CUDA "
                        "graph (the default when the inputs exceed L2; stage times always come from eager steps)")
    p.add_argument("--op", choices=("layer", "block", "dense"), default="layer",
                   help="layer: y = MoE(x) (moe_forward); block: y = h + MoE(RMSNorm(h)) (moe_forward_block); "
                        "dense: the dense SwiGLU FFN d -> 18432 -> d at the workload's T (moe_dense_ffn)")
    args = p.parse_args()
    if args.op != "layer" and args.impl == "reference":
        p.error("the reference arm times the layer")
    wl = WORKLOADS[args.workload]
    if args.tokens > 0:
        wl = wl.with_T(args.tokens)
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.op == "dense":
        return run_dense(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
