#!/usr/bin/env python3
"""Benchmark of the int4 expert-FFN MoE layer forward (sigmoid+bias router,
top-k, int4 SwiGLU experts, shared expert, weighted combine) on B200.

Default workload: the Nano decode stack -- 23 stacked MoE layers (hidden 1024,
64 experts, top-2, routed intermediate 512, shared intermediate 2048), each
layer adding its input (x_{l+1} = x_l + MoE_l(x_l)), at T=64 tokens, run as
ONE moe_stack_forward call (the fused stack kernel), with the sweep over the
decode and speculative-verify sizes T in {1,2,3,4,16,64} (fused kernel and
per-layer kernel sequences) reported beside it.  One step = one pass of the
whole layer stack over one batch of synthetic tokens.  The metric counts one
token passing through one MoE layer as one token (tokens/s = T*layers/s).
The line also carries the other workloads (one Nano layer at T=16, Nano
prefill at T=4096, Zipf routing at T=16384, the large layer at T=1, 32 and
512), each timed through the public API with its own clock record.

Timing: W warm-up steps, then exactly K timed steps bracketed by a barrier
and a device synchronize; each step is timed with CUDA events on the stream
that runs it, and L2 is flushed (a 256 MiB write) between steps, outside the
timed events.  Four different input batches rotate, so the routing changes
from step to step.  The step is replayed as a CUDA graph of the library's
C-ABI call(s).  The fused kernel is the whole step, so its roofline uses the
step's median time; for the per-layer kernel sequences an instrumented eager
pass records the library's per-stage events to time each kernel.

--impl reference times the CPU oracle (plain C, double precision, one core)
on a bounded sample of the same workload.

Multi-GPU (torchrun, N>1): independent replicas, one per GPU, no collective on
the data path (the layer has no exchange step); the time is the max over ranks.
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "MoE-layer tokens/s; achieved HBM GB/s (decode) and TFLOPS (prefill) vs roofline"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20
N_BATCHES = 4


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="nano_decode_stack", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None, help="T (default: the workload's largest)")
    ap.add_argument("--no-sweep", action="store_true", help="skip the per-T sweep of the decode stack")
    ap.add_argument("--no-graph", action="store_true", help="launch the C-ABI calls directly")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads (prefill, Zipf, large layer) reported beside the decode stack")
    ap.add_argument("--per-layer", action="store_true",
                    help="time the stack as one moe_layer_forward call per layer, whatever the library's choice")
    ap.add_argument("--fused", action="store_true",
                    help="time the fused stack kernel wherever it serves the call (MOE_STACK_FUSED), whatever the "
                         "library's choice")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lookahead", action="store_true",
                    help="fused kernel with its L2 prefetch hints (MOE_LOOKAHEAD; the output is the same)")
    ap.add_argument("--trace", action="store_true",
                    help="add the fused kernel's per-phase timeline (MOE_TRACE stamps) to the line")
    return ap.parse_args()


# --------------------------------------------------------------------------- peaks

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region: through
    NVML every 2 ms on the GPU this process uses (matched by PCI bus id), else
    through nvidia-smi every 200 ms.  Reading only; no setting is changed."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}
    PERIOD_S = 0.002

    def __init__(self, index: int, pci_bus_id: str = None):
        self.index = index
        self.pci_bus_id = pci_bus_id
        self.proc = None
        self.nvml = None
        self.lines = []
        self.samples = []  # (sm_mhz, max_mhz, reason bits)
        self.stop = threading.Event()

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            if self.pci_bus_id:
                h = pynvml.nvmlDeviceGetHandleByPciBusId(self.pci_bus_id.encode())
            else:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.nvml = (pynvml, h)
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _poll(self):
        nv, h = self.nvml
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self.stop.is_set():
            try:
                self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                     float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)),
                                     int(reasons(h))))
            except Exception:
                return
            self.stop.wait(self.PERIOD_S)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        self.stop.set()
        if self.nvml is not None:
            self.t.join(timeout=5)
            try:
                self.nvml[0].nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for f, m, bits in self.samples:
            sm.append(f)
            mx.append(m)
            reasons.update(n for n, b in self.REASON_BITS.items() if bits & b)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def pci_bus_id(device) -> str:
    """NVML-style PCI bus id of a torch CUDA device, or None."""
    try:
        pr = torch.cuda.get_device_properties(device)
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except Exception:
        return None


# --------------------------------------------------------------------------- work accounting

def step_bytes_flops(shape, T, uniq_per_layer, wbits=4):
    """Algorithmic bytes and flops of one pass over the layers.

    bytes: router W + bias, shared-expert weights + scales, every touched
    routed expert's weights + scales, x in and out (bf16).  Scratch excluded.
    flops: 2*T*E*H + 6*T*K*H*I + 6*T*H*Is per layer."""
    lb = workloads.layer_weight_bytes(shape, wbits)
    H, E, K, I, Is = shape.H, shape.E, shape.K, shape.I, shape.Is
    nbytes = 0
    for u in uniq_per_layer:
        nbytes += lb["router"] + lb["shared"] + u * lb["expert"] + 2 * T * H * 2
    flops = len(uniq_per_layer) * (2 * T * E * H + 6 * T * K * H * I + 6 * T * H * Is)
    return nbytes, flops


def stage_work(stage, shape, T, uniq, wbits=4):
    """Algorithmic (bytes, flops) of one launch of a layer stage.

    gate_up: the w13 codes + scales of every touched routed expert and of the
    shared expert, the activations read once, h written; 2 flop per MAC of
    gate and up.  down: the w2 codes + scales, h read, y (f32) written.  Only
    real tokens count (no tile padding), scratch traffic beyond that is not
    algorithmic."""
    H, K, I, Is = shape.H, shape.K, shape.I, shape.Is
    cb = 8 // wbits  # code elements per byte
    if stage == "gate_up":
        per_expert = 2 * I * H // cb + 2 * I * 4
        shared = (2 * Is * H // cb + 2 * Is * 4) if Is else 0
        nbytes = uniq * per_expert + shared + T * H * 2 + T * K * I * 2 + T * Is * 2
        flops = 4 * T * K * H * I + 4 * T * H * Is
    elif stage == "down":
        per_expert = H * I // cb + H * 4
        shared = (H * Is // cb + H * 4) if Is else 0
        nbytes = uniq * per_expert + shared + T * K * I * 2 + T * Is * 2 + (T * K + (T if Is else 0)) * H * 4
        flops = 2 * T * K * H * I + 2 * T * H * Is
    else:
        raise ValueError(stage)
    return nbytes, flops


# --------------------------------------------------------------------------- our arm

class Runner:
    """A workload's weights and the buffers of one T, with one step = one pass
    of every layer over one batch: ONE moe_stack_forward call, either the
    fused stack kernel (mode "fused") or one layer call per layer inside the
    library (mode "per_layer"; the instrumented pass and the routing count
    call moe_layer_forward per layer themselves)."""

    def __init__(self, moe, wl, T, device, stacked, mode, extra_flags=0):
        self.moe, self.wl, self.T, self.device, self.mode = moe, wl, T, device, mode
        self.shape = wl.shape
        self.L = wl.layers
        self.stacked = stacked
        self.layers = [{k: v[l] for k, v in stacked.items()} for l in range(self.L)]
        self.xs = [workloads.make_x(wl.shape, T, wl.wid, batch=b, device=device) for b in range(N_BATCHES)]
        self.outs = torch.empty((self.L, T, wl.shape.H), dtype=torch.bfloat16, device=device)
        self.flags = (moe.MOE_ADD_RESIDUAL if wl.residual else 0) | extra_flags
        self.flags |= moe.MOE_WEIGHTS_INT8 if wl.wbits == 8 else 0
        if mode == "fused":  # the fused kernel wherever it serves the call (not the library's default choice)
            self.flags |= moe.MOE_STACK_FUSED
            n = moe.stack_workspace_bytes(wl.shape, T, self.L, self.flags)
            self.ws = torch.empty(n, dtype=torch.uint8, device=device)
        else:
            self.ws = moe.new_workspace(wl.shape, T, device, self.flags)

    def run(self, b, x=None, stage_events=None, topk_idx=None):
        inp = self.xs[b] if x is None else x
        if self.mode == "fused":
            self.moe.stack_forward(inp, self.stacked, self.shape, outs=self.outs, workspace=self.ws, flags=self.flags,
                                   topk_idx=topk_idx)
        elif stage_events is None and topk_idx is None:
            self.moe.stack_forward(inp, self.stacked, self.shape, outs=self.outs, workspace=self.ws, flags=self.flags)
        else:
            # a per-layer slice of [L][T][K] need not be 16-byte aligned: one [T][K] buffer per call
            one = None if topk_idx is None else torch.empty_like(topk_idx[0])
            for l, layer in enumerate(self.layers):
                ev = None if stage_events is None else stage_events[l]
                self.moe.layer_forward(inp, layer, self.shape, out=self.outs[l], workspace=self.ws, flags=self.flags,
                                       stage_events=ev, topk_idx=one)
                if one is not None:
                    topk_idx[l].copy_(one)
                inp = self.outs[l]
        return self.outs[self.L - 1]

    def routing_unique(self):
        """Touched routed experts per (batch, layer), from the library's top-k output."""
        idx = torch.empty((self.L, self.T, self.shape.K), dtype=torch.int32, device=self.device)
        out = []
        for b in range(N_BATCHES):
            self.run(b, topk_idx=idx)
            out.append([int(torch.unique(idx[l]).numel()) for l in range(self.L)])
        torch.cuda.synchronize()
        return out

    def launches_per_step(self):
        if self.mode == "fused":
            return 1
        return self.moe.kernel_launches(self.shape, self.T, self.flags) * self.L

    def path(self):
        return self.moe.layer_path(self.shape, self.T, self.flags)


def make_events(n):
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()
    return evs


def timed_steps(runner, steps, warmup, use_graph, flush, instrumented=False, dist_barrier=None):
    """Returns (per-step ms list, per-stage ms sums per step).

    Each step is timed with CUDA events on the stream that runs it; the L2
    flush runs before each step, outside the events.  instrumented=True (per
    layer mode only): the library records its per-stage events around every
    kernel; events recorded inside a captured graph cannot be timed, so this
    pass launches the C-ABI calls directly, behind a GPU sleep long enough for
    the whole step to be queued first, so that the brackets hold device time
    and not host launch latency (but the kernels no longer overlap their
    neighbours' tails, so a kernel's time there is an upper bound)."""
    L = runner.L
    stage_ev = [make_events(8) for _ in range(L)] if instrumented else None
    if instrumented:
        use_graph = False
    torch.cuda.synchronize()
    graphs = None
    if use_graph:
        graphs = []
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for b in range(N_BATCHES):  # eager warm-up before capture
                runner.run(b)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for b in range(N_BATCHES):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                runner.run(b)
            graphs.append(g)
        torch.cuda.synchronize()

    def one(b):
        if graphs is not None:
            graphs[b].replay()
        else:
            runner.run(b, stage_events=stage_ev)

    for i in range(warmup):
        flush.zero_()
        one(i % N_BATCHES)
    torch.cuda.synchronize()
    if dist_barrier:
        dist_barrier()
    torch.cuda.synchronize()
    st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    stage_ms = []
    for i in range(steps):
        flush.zero_()
        if instrumented:
            torch.cuda._sleep(20_000_000)
        st[i].record()
        one(i % N_BATCHES)
        en[i].record()
        if instrumented:
            en[i].synchronize()
            stage_ms.append([sum(stage_ev[l][2 * s].elapsed_time(stage_ev[l][2 * s + 1]) for l in range(L))
                             for s in range(4)])
    torch.cuda.synchronize()
    if dist_barrier:
        dist_barrier()
    torch.cuda.synchronize()
    step_ms = [st[i].elapsed_time(en[i]) for i in range(steps)]
    del graphs
    return step_ms, stage_ms


def e2e_steps(runner, steps, warmup, flush, dist_barrier=None):
    """Same step through the public API with host buffers: pinned host x ->
    device, the step (a CUDA graph of the C-ABI call(s)), the last layer's
    output device -> pinned host."""
    T, H = runner.T, runner.shape.H
    host_x = [runner.xs[b].cpu().pin_memory() for b in range(N_BATCHES)]
    host_out = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(runner.xs[0])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        runner.run(0, x=x_dev)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out_dev = runner.run(0, x=x_dev)
    torch.cuda.synchronize()

    def one(b):
        x_dev.copy_(host_x[b], non_blocking=True)
        g.replay()
        host_out.copy_(out_dev, non_blocking=True)

    for i in range(warmup):
        flush.zero_()
        one(i % N_BATCHES)
    torch.cuda.synchronize()
    if dist_barrier:
        dist_barrier()
    st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        st[i].record()
        one(i % N_BATCHES)
        en[i].record()
    torch.cuda.synchronize()
    if dist_barrier:
        dist_barrier()
    ms = [st[i].elapsed_time(en[i]) for i in range(steps)]
    del g
    return ms, T * H * 2, T * H * 2


def host_cpu():
    """CPU model and logical CPU count of the host (for the CPU baseline)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


class pinned_to_one_core:
    """Runs the block on one host core (the first this process may use), as the
    CPU baseline plan asks (taskset -c <core>); restores the affinity after."""

    def __enter__(self):
        self.old = None
        self.core = None
        try:
            self.old = os.sched_getaffinity(0)
            self.core = min(self.old)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            pass
        return self

    def __exit__(self, *a):
        if self.old is not None:
            try:
                os.sched_setaffinity(0, self.old)
            except OSError:
                pass


def cpu_baseline_sample(runner, budget_s=15.0):
    """The oracle (single-threaded C, f64) on a bounded sample of the step:
    the first tokens of batch 0 through every layer, each layer fed the GPU's
    bf16 input of that layer, pinned to one host core.  Returns (tokens/s
    counting token-layers, the sample, the core)."""
    import oracle
    shape = runner.shape
    with torch.no_grad():
        runner.run(0)
        torch.cuda.synchronize()
        inputs = [runner.xs[0]] + [runner.outs[l] for l in range(runner.L - 1)]
        inputs = [t.cpu() for t in inputs]
    layers_cpu = [{k: v.cpu() for k, v in layer.items()} for layer in runner.layers]
    with pinned_to_one_core() as pin:
        t0 = time.perf_counter()
        oracle.moe_tokens(inputs[0], layers_cpu[0], shape, residual=runner.wl.residual, tokens=[0])
        per = max(time.perf_counter() - t0, 1e-4)
        n_tok = int(max(1, min(runner.T, budget_s / (per * len(layers_cpu)))))
        toks = list(range(n_tok))
        t0 = time.perf_counter()
        for l, layer in enumerate(layers_cpu):
            oracle.moe_tokens(inputs[l], layer, shape, residual=runner.wl.residual, tokens=toks)
        dt = time.perf_counter() - t0
    sample = f"{n_tok} of {runner.T} tokens of one batch through all {len(layers_cpu)} layers ({dt:.1f} s)"
    return n_tok * len(layers_cpu) / dt, sample, pin.core


def captured_entry(workload: str, T: int, kernel: str):
    """The committed ncu capture of `kernel` on this workload and T
    (profiles/traffic.json), or None when there is none or the kernel's
    sources have changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entries = json.load(f)["entries"]
    except (OSError, ValueError, KeyError):
        return None
    for e in entries:
        if (e["workload"], e["T"], e["kernel"]) != (workload, T, kernel):
            continue
        h = hashlib.sha256()
        try:
            for src in e["sources"]:
                with open(os.path.join(ROOT, src), "rb") as f:
                    h.update(f.read())
        except OSError:
            return None
        return e if h.hexdigest() == e["sha256"] else None
    return None


def captured_traffic(workload: str, T: int, kernel: str):
    """DRAM bytes (read + written) per launch from the committed capture, or None."""
    e = captured_entry(workload, T, kernel)
    return int(e["read"]) + int(e["write"]) if e else None


def streaming_kernel_names(shape, T, wbits=4):
    """Gate/up and down kernels of the weight-streaming path for this shape
    and T (the library's selection: TMA-ring kernels from H = 1024 on when H,
    I and Is are multiples of 256, the tcgen05 gate/up kernel among them on
    the large-batch sequence at 12 or more picks per routed expert with int4
    codes; bulk-copy gate/up below; register-ring kernels otherwise)."""
    tma2 = shape.H >= 1024 and shape.I % 256 == 0 and shape.Is % 256 == 0
    if shape.H >= 1024 and shape.H % 256 == 0:
        tc8 = wbits == 4 and tma2 and T > 64 and T * shape.K >= 12 * shape.E
        w13 = "experts_w13_tc8_kernel" if tc8 else "experts_w13_tma_kernel"
    else:
        w13 = "experts_w13_bulk_kernel" if shape.H <= 1024 else "experts_w13_kernel"
    return w13, "experts_w2_tma_kernel" if tma2 else "experts_w2_kernel"


def max_over_ranks(values, dist, device):
    """Element-wise maximum of `values` over all ranks (the slowest rank's
    times); the values themselves for a single process (dist None)."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_throughput(world, tokens_per_step, steps, total_ms):
    """Whole-job tokens/s: every rank ran `steps` steps of `tokens_per_step`
    tokens, and the job took the slowest rank's `total_ms`."""
    return world * tokens_per_step * steps / (total_ms / 1e3)


def phase_trace(moe, runner):
    """One traced call of the fused kernel (MOE_TRACE stamps, see
    moe_stack_trace_offset).  Per layer: the critical path split into the
    router part (the last CTA done with the previous layer's down tasks ->
    every token group selected) and the expert part (selected -> the last CTA
    done with this layer's down tasks); and the steps inside them, each the
    median over the CTAs that took both of its stamps.  Medians over the
    layers, in microseconds."""
    T, L, shape = runner.T, runner.L, runner.shape
    flags = runner.flags | moe.MOE_TRACE
    ws = torch.empty(moe.stack_workspace_bytes(shape, T, L, flags), dtype=torch.uint8, device=runner.device)
    moe.stack_forward(runner.xs[0], runner.stacked, shape, outs=runner.outs, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    grid = torch.cuda.get_device_properties(runner.device).multi_processor_count
    st = moe.stack_trace(ws, shape, T, L, flags, grid).double() / 1e3  # us, 0 = not taken

    def span(s, a, b):
        ok = (s[:, a] > 0) & (s[:, b] > 0)
        return float(torch.median(s[ok, b] - s[ok, a])) if bool(ok.any()) else None

    steps = {"wait_prev_down": (0, 1), "combine": (1, 7), "router_mma": (7, 8), "count": (8, 9),
             "select": (9, 10), "quantize": (10, 11), "units_to_selected": (2, 3), "tables": (3, 4),
             "prefetch": (4, 12), "first_stage": (12, 13), "gate_up": (4, 5), "down_ready": (5, 14),
             "down_stage_h": (14, 15), "down": (5, 6)}
    rows = {k: [] for k in ["router_critical", "experts_critical", "layer", "selected_seen"] + list(steps)}
    for l in range(L):
        s = st[:, l]
        prev_end = st[:, l - 1, 6].max() if l > 0 else st[:, 0, 0][st[:, 0, 0] > 0].min()
        sel = s[:, 3][s[:, 3] > 0].min()
        end = s[:, 6].max()
        rows["router_critical"].append(float(sel - prev_end))
        rows["experts_critical"].append(float(end - sel))
        rows["layer"].append(float(end - prev_end))
        q = s[:, 11][s[:, 11] > 0]
        if q.numel():
            rows["selected_seen"].append(float(sel - q.max()))
        for k, (a_, b_) in steps.items():
            v = span(s, a_, b_)
            if v is not None:
                rows[k].append(v)
    out = {k: round(statistics.median(v), 2) for k, v in rows.items() if v}
    out["total_us"] = round(float(st[:, L, 2].max() - st[:, 0, 0][st[:, 0, 0] > 0].min()), 1)
    out["note"] = ("one traced call (L2 not flushed before it); per layer, medians over the CTAs of each step's "
                   "duration, then medians over the layers, us")
    return out


def dist_or_none(world, dist):
    return dist if world > 1 else None


def percentiles(ms):
    s = sorted(ms)
    q = lambda f: s[min(len(s) - 1, int(f * (len(s) - 1) + 0.5))]
    return {"median": round(statistics.median(s), 4), "p10": round(q(0.1), 4), "p90": round(q(0.9), 4),
            "mean": round(statistics.mean(s), 4), "n": len(s)}


def roofline_of(alg_b, alg_f, seconds, peaks, kernel, timing, traffic=None):
    """Roofline object of one kernel (or step): bound from the arithmetic
    intensity against the ridge of the measured peaks."""
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if alg_b > 0 and alg_f / alg_b >= ridge:
        achieved = alg_f / seconds / 1e12
        r = {"bound": "tensor", "kernel": kernel, "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
             "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
             "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json bf16_tflops, burst)"}
    else:
        achieved = alg_b / seconds / 1e9
        r = {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
             "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
             "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs, copy)"}
    r.update({"traffic": traffic, "alg_bytes_per_launch": int(alg_b), "alg_flops_per_launch": int(alg_f),
              "avg_launch_us": round(seconds * 1e6, 3), "timing": timing})
    return r


def with_ncu_time(r, workload, T, kernel):
    """Adds the committed ncu launch time (cold cache, serialised) of the same
    kernel, workload and T beside the live one, as a cross-check."""
    e = captured_entry(workload, T, kernel)
    r["ncu_launch_us"] = e.get("ncu_us") if e else None
    return r


def stacked_weights(moe, wl, device):
    layers = [workloads.make_layer(wl.shape, wl.wid, l, device, wl.bias_mode, wbits=wl.wbits) for l in range(wl.layers)]
    st = moe.stack_layers(layers)
    del layers
    torch.cuda.empty_cache()
    return st


def measure(runner, steps, warmup, use_graph, flush, peaks, device, barrier=None):
    """Timed steps of one runner with its clock record and work accounting."""
    uniq = runner.routing_unique()
    with ClockSampler(device.index if device.index is not None else 0, pci_bus_id(device)) as clk:
        ms, _ = timed_steps(runner, steps, warmup, use_graph, flush, dist_barrier=barrier)
    work = [step_bytes_flops(runner.shape, runner.T, uniq[i % N_BATCHES], runner.wl.wbits) for i in range(steps)]
    return {"ms": ms, "uniq": uniq, "clocks": clk.summary(), "bytes": statistics.mean(w[0] for w in work),
            "flops": statistics.mean(w[1] for w in work)}


def workload_entry(moe, wl, T, device, steps, warmup, use_graph, flush, peaks, stacked=None):
    """One extra workload: its step (all its layers) timed through the public
    API, median over the steps, with its own clock record; for the per-layer
    kernel sequences the dominant expert kernel's rate from the instrumented
    eager pass."""
    stacked = stacked if stacked is not None else stacked_weights(moe, wl, device)
    L = wl.layers
    modes = ["per_layer"]
    wflags = (moe.MOE_ADD_RESIDUAL if wl.residual else 0) | (moe.MOE_WEIGHTS_INT8 if wl.wbits == 8 else 0)
    if moe.stack_path(wl.shape, T, L, wflags | moe.MOE_STACK_FUSED) == moe.MOE_PATH_FUSED_STACK:
        modes.insert(0, "fused")
    entry = {"workload": wl.name, "T": T, "layers": L, "expert_bits": wl.wbits}
    for mode in modes:
        r = Runner(moe, wl, T, device, stacked, mode)
        m = measure(r, steps, warmup, use_graph, flush, peaks, device)
        med = statistics.median(m["ms"]) / 1e3
        d = {"ms_per_step": percentiles(m["ms"]), "tokens_per_s": round(T * L / med, 1),
             "alg_bytes_per_step": int(m["bytes"]), "alg_flops_per_step": int(m["flops"]),
             "step_roofline": roofline_of(m["bytes"], m["flops"], med, peaks, "whole step", "CUDA graph, median"),
             "clocks": m["clocks"], "gpu_launches_per_step": r.launches_per_step(),
             "path": "fused stack kernel" if mode == "fused" else
                     {moe.MOE_PATH_SMALL_BATCH: "small-batch kernels", moe.MOE_PATH_TENSOR_CORE: "tensor-core kernels",
                      moe.MOE_PATH_LARGE_STREAMING: "large-batch streaming kernels"}[r.path()]}
        if mode == "per_layer":
            _, stage_ms = timed_steps(r, max(3, steps // 2), 2, use_graph, flush, instrumented=True)
            stage_mean = [statistics.mean(s[k] for s in stage_ms) for k in range(4)]
            dom = 1 if stage_mean[1] >= stage_mean[2] else 2
            names = moe.STAGE_NAMES
            tc = r.path() == moe.MOE_PATH_TENSOR_CORE
            w13, w2 = streaming_kernel_names(wl.shape, T, wl.wbits)
            kname = (f"grouped_gemm_kernel<{dom}, {wl.wbits}>" if tc else (w13 if dom == 1 else w2))
            u = m["uniq"]
            kw = [[stage_work(names[dom], wl.shape, T, x, wl.wbits) for x in u[i % N_BATCHES]]
                  for i in range(len(stage_ms))]
            kb = statistics.mean(sum(w[0] for w in ws) for ws in kw) / L
            kf = statistics.mean(sum(w[1] for w in ws) for ws in kw) / L
            d["stages_us_per_step"] = {names[k]: round(stage_mean[k] * 1e3, 2) for k in range(4)}
            d["kernel_roofline"] = with_ncu_time(
                roofline_of(kb, kf, stage_mean[dom] / L / 1e3, peaks, kname,
                            "eager pass with per-stage events (no overlap with neighbours)",
                            captured_traffic(wl.name, T, kname)), wl.name, T, kname)
        entry[mode] = d
        del r
        torch.cuda.empty_cache()
    return entry


def run_ours(args, rank, world, device, dist):
    import int4_expert_ffn_sigmoid_b200 as moe
    wl = workloads.WORKLOADS[args.workload]
    T = args.tokens or max(wl.tokens)
    peaks = measured_peaks()
    barrier = (lambda: dist.barrier()) if world > 1 else None
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    use_graph = not args.no_graph
    stacked = stacked_weights(moe, wl, device)
    flags = (moe.MOE_ADD_RESIDUAL if wl.residual else 0) | (moe.MOE_WEIGHTS_INT8 if wl.wbits == 8 else 0)
    # the library's own choice for the call (moe_stack_path), unless a flag forces one
    choice = flags | (moe.MOE_STACK_FUSED if args.fused else 0)
    fused = (not args.per_layer) and moe.stack_path(wl.shape, T, wl.layers, choice) == moe.MOE_PATH_FUSED_STACK
    runner = Runner(moe, wl, T, device, stacked, "fused" if fused else "per_layer",
                    moe.MOE_LOOKAHEAD if (args.lookahead and fused) else 0)
    L = wl.layers

    m = measure(runner, args.steps, args.warmup, use_graph, flush, peaks, device, barrier)
    step_ms = m["ms"]
    e2e_ms, h2d, d2h = e2e_steps(runner, args.steps, args.warmup, flush, dist_barrier=barrier)
    total_ms, e2e_total, med_ms = max_over_ranks([sum(step_ms), sum(e2e_ms), statistics.median(step_ms)],
                                                 dist_or_none(world, dist), device)
    tokens_per_step = T * L
    value = job_throughput(world, tokens_per_step, args.steps, total_ms)
    e2e_value = job_throughput(world, tokens_per_step, args.steps, e2e_total)
    ms_mean = total_ms / args.steps
    step_gbs = m["bytes"] / (ms_mean / 1e3) / 1e9

    if fused:
        # one kernel per step: the step's events bracket it (and the counters'
        # memset that precedes it, about 1-2 us)
        roofline = with_ncu_time(
            roofline_of(m["bytes"], m["flops"], med_ms / 1e3, peaks, "decode_stack_kernel",
                        "CUDA graph step (memset + the one kernel), median over the timed steps",
                        captured_traffic(wl.name, T, "decode_stack_kernel")), wl.name, T, "decode_stack_kernel")
        stages = None
    else:
        _, stage_ms = timed_steps(runner, args.steps, 2, use_graph, flush, instrumented=True)
        stage_mean = [statistics.mean(s[k] for s in stage_ms) for k in range(4)]
        names = moe.STAGE_NAMES
        dom = 1 if stage_mean[1] >= stage_mean[2] else 2
        tc = runner.path() == moe.MOE_PATH_TENSOR_CORE
        w13, w2 = streaming_kernel_names(wl.shape, T, wl.wbits)
        kname = f"grouped_gemm_kernel<{dom}, {wl.wbits}>" if tc else (w13 if dom == 1 else w2)
        kw = [[stage_work(names[dom], wl.shape, T, u, wl.wbits) for u in m["uniq"][i % N_BATCHES]]
              for i in range(len(stage_ms))]
        roofline = with_ncu_time(
            roofline_of(statistics.mean(sum(w[0] for w in ws) for ws in kw) / L,
                        statistics.mean(sum(w[1] for w in ws) for ws in kw) / L,
                        stage_mean[dom] / L / 1e3, peaks, kname,
                        "eager pass with per-stage events (no overlap with neighbours)",
                        captured_traffic(wl.name, T, kname)), wl.name, T, kname)
        stages = {names[k]: round(stage_mean[k] * 1e3, 2) for k in range(4)}

    trace = phase_trace(moe, runner) if (args.trace and fused) else None

    sweep = {}
    if wl.name == "nano_decode_stack" and not args.no_sweep:
        for Ts in wl.tokens:
            row = {}
            for mode in ("fused", "per_layer"):
                if mode == "fused" and \
                        moe.stack_path(wl.shape, Ts, L, flags | moe.MOE_STACK_FUSED) != moe.MOE_PATH_FUSED_STACK:
                    continue
                r = runner if (Ts == T and mode == runner.mode) else Runner(moe, wl, Ts, device, stacked, mode)
                ms = m if r is runner else measure(r, max(10, args.steps // 2), 3, use_graph, flush, peaks, device)
                med = statistics.median(ms["ms"])
                row[mode] = {"ms_per_step": round(med, 4), "tokens_per_s": round(Ts * L / (med / 1e3), 1),
                             "step_gbs": round(ms["bytes"] / (med / 1e3) / 1e9, 1),
                             "step_hbm_frac": round(ms["bytes"] / (med / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                             "sm_mhz": ms["clocks"]["sm_mhz"], "reasons": ms["clocks"]["reasons"]}
                if r is not runner:
                    del r
                    torch.cuda.empty_cache()
            sweep[str(Ts)] = row

    extra = None
    if world == 1 and not args.no_workloads and wl.name == "nano_decode_stack":
        extra = []
        steps = max(10, args.steps)
        for name, Ts_list in (("nano_layer_t16", (16,)), ("nano_prefill_t4096", (4096,)),
                              ("nano_prefill_t4096_int8", (4096,)), ("nano_zipf_t16384", (16384,)),
                              ("large_layer", (1, 32, 512))):
            w2l = workloads.WORKLOADS[name]
            st = stacked_weights(moe, w2l, device)
            for Ts in Ts_list:
                extra.append(workload_entry(moe, w2l, Ts, device, steps, 3, use_graph, flush, peaks, st))
            del st
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, core = cpu_baseline_sample(runner)
        cpu = {"value": round(v, 2), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
               "pinned_core": core, **host_cpu()}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_mean, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "int8" if runner.mode == "fused" or runner.path() != moe.MOE_PATH_TENSOR_CORE else "bf16",
        "dtype_note": "weight-streaming arithmetic: int4 codes as int8, activations as two int8 parts, exact int32 "
                      "products, f32 router, scales and sums, bf16 in and out",
        "data": "synthetic",
        "config": {"workload": wl.name, "layers": L, "T": T, "H": wl.shape.H, "E": wl.shape.E,
                   "K": wl.shape.K, "I": wl.shape.I, "Is": wl.shape.Is, "tokens_counted": "T*layers per step",
                   "path": "fused stack kernel (moe_stack_forward)" if fused else "one moe_layer_forward per layer",
                   "l2": "flushed between steps (256 MiB write, outside the timed events)",
                   "inputs": f"{N_BATCHES} rotating batches", "cuda_graph": use_graph,
                   "parallelism": "replicas" if world > 1 else "single"},
        "timing": {"ms_per_step": percentiles(step_ms)},
        "step_hbm": {"achieved_gbs": round(step_gbs, 1), "frac": round(step_gbs / peaks["hbm_gbs"], 4),
                     "alg_bytes_per_step": int(m["bytes"]), "tflops": round(m["flops"] / (ms_mean / 1e3) / 1e12, 3)},
        "stages_us_per_step": stages,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": runner.launches_per_step() * args.steps,
        "clocks": m["clocks"],
        "sweep": sweep or None,
        "trace": trace,
        "workloads": extra,
    }
    return line


# --------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step is a bounded sample of
    the workload (the first tokens of a batch through every layer, the oracle
    chaining its own outputs rounded to bf16 as the next layer's input), on
    one pinned host core."""
    import oracle
    if rank != 0:
        return None
    wl = workloads.WORKLOADS[args.workload]
    T = args.tokens or max(wl.tokens)
    layers = [workloads.make_layer(wl.shape, wl.wid, l, "cpu", wl.bias_mode, wbits=wl.wbits) for l in range(wl.layers)]
    xs = [workloads.make_x(wl.shape, T, wl.wid, batch=b, device="cpu") for b in range(N_BATCHES)]
    n_tok = min(T, 4)

    def step(i):
        x = xs[i % N_BATCHES][:n_tok].contiguous()
        for layer in layers:
            r = oracle.moe_tokens(x, layer, wl.shape, residual=wl.residual)
            x = torch.from_numpy(r["out"]).to(torch.bfloat16)

    with pinned_to_one_core() as pin:
        for i in range(args.warmup):
            step(i)
        t0 = time.perf_counter()
        for i in range(args.steps):
            step(i)
        dt = time.perf_counter() - t0
    value = n_tok * wl.layers * args.steps / dt
    sample = f"{n_tok} of {T} tokens per step through all {wl.layers} layers"
    return {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "layers": wl.layers, "T": T, "H": wl.shape.H, "E": wl.shape.E,
                       "K": wl.shape.K, "I": wl.shape.I, "Is": wl.shape.Is, "tokens_counted": "T*layers per step"},
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                             "pinned_core": pin.core, **host_cpu()},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    dist = None
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    try:
        line = run_ours(args, rank, world, device, dist)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
