#!/usr/bin/env python
"""Throughput of the B200 Mixtral sparse-MoE layer (route -> dispatch -> experts -> combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|skew|quarter|tiny]
                    [--impl ours|reference]

One step = one forward of the whole layer over one batch of T synthetic tokens
(Mixtral 8x7B shapes: d=4096, d_ff=14336, E=8, k=2), inputs resident in HBM.
Timing: CUDA events on the launching stream around each step, W warm-up steps,
512 MiB written between timed steps to flush the 126 MB L2; the per-step device
time excludes the flush.  N > 1 (torchrun): every rank runs an independent
replica on its own GPU (no collective on the data path); the reported time is
the max over ranks and `value` counts the tokens of all ranks.

`--impl reference` times the CPU oracle (oracle/, plain C, fp64) on a bounded
sample of the same workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; % of BF16 TC peak (prefill), % of HBM GB/s (decode)"
WORKLOAD_NAMES = {
    "prefill": "mixtral-8x7b-moe-prefill T=4096",
    "decode": "mixtral-8x7b-moe-decode T=16",
    "skew": "mixtral-8x7b-moe-prefill-skewed T=16384",
    "quarter": "quarter-width-moe T=1024 d=1024 d_ff=3584",
    "tiny": "tiny-moe T=64 d=128 d_ff=256",
}
FLUSH_BYTES = 512 << 20
SETTLE_S = 1.0  # GPU idle before a secondary workload or the end-to-end queue is timed
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
KERNEL_SOURCES = ["sparse_mixture_experts_05_b200/csrc/expert_gemm.cu",
                  "sparse_mixture_experts_05_b200/csrc/sm100.cuh",
                  "sparse_mixture_experts_05_b200/csrc/common.cuh",
                  "sparse_mixture_experts_05_b200/csrc/combine_math.cuh"]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill", choices=list(WORKLOAD_NAMES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the extras and the decode, skew, quarter and tiny objects of the "
                         "prefill run")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (smaller cases for profiler captures)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (smaller cases for profiler captures)")
    ap.add_argument("--vs-cublas", action="store_true",
                    help="instead of the step: time the expert GEMMs against cuBLAS batched "
                         "bf16 GEMMs of the same shapes (equal rows per expert), alternating")
    ap.add_argument("--block-vs-plain", action="store_true",
                    help="instead of the step: the block forward (RMSNorm inside the router, "
                         "residual in the combine) and the plain layer on the block's own "
                         "normalised rows, alternating (a short run for profiler launch lists)")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


def load_peaks():
    """The measured copy bandwidth and bf16 GEMM rates of this machine's B200s from
    MEASURED_PEAKS.json (hbm_gbs, bf16_tflops, bf16_tflops_sustained), each
    missing or non-numeric entry replaced by the earlier measurement in
    FALLBACK_PEAKS; the second value says which ("measured", "partly measured",
    "fallback")."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peaks = dict(FALLBACK_PEAKS)
    try:
        with open(path) as f:
            found = json.load(f)
    except (OSError, ValueError):
        return peaks, "fallback"
    got = 0
    for key in FALLBACK_PEAKS:
        v = found.get(key) if isinstance(found, dict) else None
        if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
            peaks[key] = float(v)
            got += 1
    if got == len(FALLBACK_PEAKS):
        return peaks, "measured"
    return peaks, ("partly measured" if got else "fallback")


def source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload):
    """DRAM bytes per launch of the expert kernel from the committed ncu summary, when it
    was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "expert_gemm_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("kernel_source_sha") != source_hash():
        return None
    return t.get("per_step_bytes", {}).get(workload)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs: through
    NVML every 2 ms from a thread (a timed region of ten prefill steps lasts about
    22 ms), else through nvidia-smi every 200 ms.  Reads only; changes nothing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.002

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.nvml = None
        self.handle = None
        self.samples = []
        self.done = threading.Event()

    _handles = {}  # gpu index -> (pynvml, handle), looked up once per process

    @classmethod
    def prepare(cls, gpu_index: int):
        try:
            cls(gpu_index)._nvml_handle()
        except Exception:
            pass

    def _nvml_handle(self):
        if self.gpu_index in ClockSampler._handles:
            return ClockSampler._handles[self.gpu_index]
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            prop = torch.cuda.get_device_properties(self.gpu_index)
            bus = "%08x:%02x:%02x.0" % (prop.pci_domain_id, prop.pci_bus_id, prop.pci_device_id)
            got = (pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus))
        except Exception:
            got = (pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu_index))
        ClockSampler._handles[self.gpu_index] = got
        return got

    def start(self):
        try:
            self.nvml, self.handle = self._nvml_handle()
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._nvml_loop, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _nvml_loop(self):
        n = self.nvml
        while True:
            try:
                sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                why = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((float(sm), int(why)))
            except Exception:
                pass
            if self.done.wait(self.PERIOD_S):
                return

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    @staticmethod
    def reasons_of(bits: int):
        """Names of the throttle reasons in an NVML clock-event bit mask (the ones the
        measurement rules look at)."""
        named = [(0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x20, "sw_thermal_slowdown"),
                 (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown")]
        return [name for bit, name in named if bits & bit]

    def stop(self):
        if self.nvml is not None:
            self.done.set()
            if self.thread:
                self.thread.join(timeout=2)
            try:
                smax = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
            except Exception:
                smax = None
            sm = [c for c, _ in self.samples]
            reasons = set()
            for _, bits in self.samples:
                reasons.update(self.reasons_of(bits))
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                    "reasons": sorted(reasons), "samples": len(sm),
                    "sampler": f"NVML every {self.PERIOD_S * 1000:.0f} ms during the timed region"}
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
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "sampler": "nvidia-smi every 200 ms"}


# ---------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if __import__("torch").cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
        pg = dist
    return world, rank, local, pg


def reduce_max(pg, value: float, device) -> float:
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, device):
    if pg is None:
        return
    import torch
    t = torch.zeros(1, device=device)
    pg.all_reduce(t)


# ---------------------------------------------------------------- our arm
def algorithmic(shape, counts):
    T, d, d_ff, E, k = shape
    R = T * k
    flops_experts = 6 * R * d * d_ff
    flops_router = 2 * T * d * E
    touched = sum(1 for c in counts if c > 0)
    weight_bytes = touched * 3 * d * d_ff * 2
    return {
        "flops_gemm1": 4 * R * d * d_ff,
        "flops_gemm2": 2 * R * d * d_ff,
        "flops_total": flops_experts + flops_router,
        "bytes_expert_weights": weight_bytes,
        # bytes each memory-bound kernel must move at least once
        "bytes_router": T * d * 2 + d * E * 2 + T * k * 8,
        "bytes_dispatch": T * k * 4 * 3 + T * d * 2 + R * d * 2,
        "bytes_combine": R * d * 4 + T * d * 2 + T * k * 8,
        # decode: the experts' weights plus their activations
        "bytes_experts_decode": weight_bytes + R * d * 2 + R * d_ff * 2 * 2 + R * d * 4,
    }


def workload(name, tokens=None, experts=None):
    import dataclasses

    from sparse_mixture_experts_05_b200.inputs import WORKLOADS
    w = WORKLOADS[name]
    if tokens is not None:
        w = dataclasses.replace(w, T=tokens)
    if experts is not None:
        w = dataclasses.replace(w, E=experts)
    return w


def workload_label(a):
    label = WORKLOAD_NAMES[a.workload]
    if a.tokens is not None or a.experts is not None:
        w = workload(a.workload, a.tokens, a.experts)
        label += f" (profiling override: T={w.T} E={w.E})"
    return label


def time_workload(name, steps, warmup, device, rank, tokens=None, experts=None):
    import torch

    import sparse_mixture_experts_05_b200 as moe
    from sparse_mixture_experts_05_b200.inputs import make_inputs

    w = workload(name, tokens, experts)
    inp = make_inputs(w.T, w.d, w.d_ff, w.E, w.k, w.seed, bias=w.skew_bias, device=device)
    shape = inp["shape"]
    x, Wg, bias, W1, W3, W2 = (inp[key] for key in ("x", "Wg", "bias", "W1", "W3", "W2"))
    ws = moe.workspace(moe.moe_forward_workspace_bytes(shape), device)
    y = torch.empty(w.T, w.d, dtype=torch.bfloat16, device=device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    n_ev = len(moe.binding.PROFILE_EVENTS)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    for row in events:
        for ev in row:
            ev.record()
    warm = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for ev in warm:
        ev.record()
    for _ in range(warmup):
        moe.moe_forward_profiled(shape, x, Wg, bias, W1, W3, W2, warm, y=y, ws=ws)
    torch.cuda.synchronize()
    status = moe.moe_read_device_status(ws)
    if status != moe.MOE_OK:
        raise RuntimeError(f"device status after warm-up: {moe.status_string(status)}")
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=device)
    moe.moe_forward(shape, x, Wg, bias, W1, W3, W2, y=y, idx_out=idx, ws=ws)
    counts = torch.bincount(idx.flatten().long(), minlength=w.E).tolist()

    plain = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(steps)]

    def run_plain(i):
        plain[i][0].record()
        moe.moe_forward(shape, x, Wg, bias, W1, W3, W2, y=y, ws=ws)
        plain[i][1].record()

    return dict(inp=inp, shape=shape, ws=ws, y=y, flush=flush, events=events, counts=counts,
                plain=plain, run_plain=run_plain,
                run=lambda i: moe.moe_forward_profiled(shape, x, Wg, bias, W1, W3, W2, events[i],
                                                       y=y, ws=ws))


def timed_loop(ctx, steps, pg, device, clock, profiled):
    """K timed steps, L2 flushed before each.  profiled=False: each step is one
    moe_forward between two events (the step time).  profiled=True: each step is
    moe_forward_profiled, whose seven events split the step by kernel."""
    import torch
    barrier(pg, device)
    torch.cuda.synchronize()
    if clock is not None:
        clock.start()
    outer0 = torch.cuda.Event(enable_timing=True)
    outer1 = torch.cuda.Event(enable_timing=True)
    outer0.record()
    run = ctx["run"] if profiled else ctx["run_plain"]
    for i in range(steps):
        ctx["flush"].fill_(i & 0xFF)
        run(i)
    outer1.record()
    torch.cuda.synchronize()
    barrier(pg, device)
    clocks = clock.stop() if clock is not None else None
    parts = {}
    if profiled:
        import sparse_mixture_experts_05_b200 as moe
        ev = ctx["events"]
        step_ms = [ev[i][0].elapsed_time(ev[i][6]) for i in range(steps)]
        names = moe.binding.PROFILE_EVENTS
        for j in range(1, len(names)):
            parts[names[j]] = sum(ev[i][j - 1].elapsed_time(ev[i][j]) for i in range(steps)) / steps
    else:
        step_ms = [a.elapsed_time(b) for a, b in ctx["plain"]]
    return step_ms, parts, outer0.elapsed_time(outer1), clocks


def extras_loop(ctx, steps, device, local):
    """The widened entry points on the same batch, interleaved step by step with
    the plain layer so that all see the same clocks and power state (L2 flushed
    before every call, clocks sampled throughout): the block with its edges,
    the layer with expert biases, and the load-balancing term on the router's
    logits.  The order of the five calls rotates by one every step, so each
    call runs in each place equally often over whole rotations (at least 30
    steps) and no call always follows the same one.  Reports each one's mean
    time and
    its difference from the plain layer as the mean over the steps of the two
    calls' difference within a step (calls of one step see the same clock,
    which drifts as the GPU heats)."""
    import torch

    import sparse_mixture_experts_05_b200 as moe
    from sparse_mixture_experts_05_b200.inputs import expert_biases
    inp = ctx["inp"]
    shape = ctx["shape"]
    T, d, d_ff, E, k = shape
    x, Wg, bias, W1, W3, W2 = (inp[key] for key in ("x", "Wg", "bias", "W1", "W3", "W2"))
    gen = torch.Generator(device=device)
    gen.manual_seed(5)
    gamma = (1 + 0.2 * torch.randn(d, generator=gen, device=device)).to(torch.bfloat16)
    eb = expert_biases(E, d, d_ff, seed=6, device=device)
    ws_b = moe.workspace(moe.moe_block_workspace_bytes(shape), device)
    H = torch.empty(T, d, dtype=torch.bfloat16, device=device)
    idx, _, logits = moe.moe_route(shape, x, Wg, bias, want_logits=True)
    # the block's normalised rows u (left in its workspace for the scatter): the
    # plain layer on u routes exactly as the block does, so block - plain-on-u
    # is the cost of the edges alone (RMSNorm inside the router, residual in
    # the combine) with the same expert loads and GEMM tiles
    moe.moe_block_forward(shape, x, gamma, Wg, bias, W1, W3, W2, H=H, ws=ws_b)
    off = moe.moe_forward_workspace_bytes(shape)
    u = ws_b[off:off + T * d * 2].view(torch.bfloat16).view(T, d).clone()
    calls = {
        "plain_ms": lambda: moe.moe_forward(shape, x, Wg, bias, W1, W3, W2, y=ctx["y"],
                                            ws=ctx["ws"]),
        "plain_on_u_ms": lambda: moe.moe_forward(shape, u, Wg, bias, W1, W3, W2, y=ctx["y"],
                                                 ws=ctx["ws"]),
        "block_forward_ms": lambda: moe.moe_block_forward(shape, x, gamma, Wg, bias, W1, W3, W2,
                                                          H=H, ws=ws_b),
        "forward_bias_ms": lambda: moe.moe_forward_bias(shape, x, Wg, bias, W1, W3, W2, eb,
                                                        y=ctx["y"], ws=ctx["ws"]),
        "aux_loss_ms": lambda: moe.moe_aux_loss(shape, logits, idx),
    }
    for call in calls.values():
        for _ in range(3):
            call()
    torch.cuda.synchronize()
    times = {name: [] for name in calls}
    clock = ClockSampler(local)
    clock.start()
    names = list(calls)
    n_steps = -(-max(steps, 30) // len(names)) * len(names)
    for i in range(n_steps):
        for j in range(len(names)):
            name = names[(i + j) % len(names)]
            call = calls[name]
            ctx["flush"].fill_(i & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            e1.synchronize()
            times[name].append(e0.elapsed_time(e1))
    clocks = clock.stop()
    if moe.moe_read_device_status(ws_b) != moe.MOE_OK:
        raise RuntimeError("device status error in the block forward")
    out = {name: round(statistics.mean(v), 4) for name, v in times.items()}

    def paired(a, b):
        return round(statistics.mean(x - y for x, y in zip(times[a], times[b])), 4)
    out["block_minus_plain_on_u_ms"] = paired("block_forward_ms", "plain_on_u_ms")
    out["bias_minus_plain_ms"] = paired("forward_bias_ms", "plain_ms")
    out["steps"] = len(times["plain_ms"])
    out["clocks"] = clocks
    out["note"] = ("same batch, calls interleaved step by step (plain, plain on u, block, bias, "
                   "aux); block = RMSNorm inside the router + layer + residual in the combine, "
                   "gamma ~ 1 + 0.2 N(0, 1); plain on u = the layer on the block's own "
                   "normalised rows (same routing and GEMM tiles as the block); bias = expert "
                   "Linear biases b1, b3, b2; aux = load-balancing term over the T x E logits; "
                   "order rotated every step; *_minus_* = mean over the steps of the "
                   "difference within a step")
    return out


def graph_step_ms(ctx, steps):
    """The step replayed from a CUDA graph of one moe_forward (captured once),
    the L2 flushed before each replay, each replay between two events with the
    host waiting for it: the device time of the layer without the host's
    per-launch work, which the eager steps of a sub-0.1 ms workload can carry
    (the host issues each eager step's six launches through the Python binding
    while the device waits).  Returns (median, mean) in ms."""
    import torch

    import sparse_mixture_experts_05_b200 as moe
    inp = ctx["inp"]
    shape = ctx["shape"]
    args = tuple(inp[key] for key in ("x", "Wg", "bias", "W1", "W3", "W2"))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        moe.moe_forward(shape, *args, y=ctx["y"], ws=ctx["ws"])
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        moe.moe_forward(shape, *args, y=ctx["y"], ws=ctx["ws"])
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    ms = []
    for i in range(steps):
        ctx["flush"].fill_(i & 0xFF)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        b.synchronize()
        ms.append(a.elapsed_time(b))
    if moe.moe_read_device_status(ctx["ws"]) != moe.MOE_OK:
        raise RuntimeError("device status error in the graph replays")
    del graph
    return statistics.median(ms), statistics.mean(ms)


def secondary_workload(name, steps, warmup, device, rank, local, pg, peaks):
    """A second workload timed like the main one (plain pass with clocks, then the
    profiled pass for the kernel split) and summarised as an object of the line.
    It starts after SETTLE_S seconds with the GPU idle, so that it runs in its own
    power state rather than in the tail of the power limiter's response to the
    workload before it (the decode batch, which streams weights, measured 0.49-0.50
    ms at 1387 MHz right after the prefill queue and 0.44 ms at full clock)."""
    w_steps = steps
    import torch
    torch.cuda.synchronize()
    time.sleep(SETTLE_S)
    ctx = time_workload(name, w_steps, warmup, device, rank)
    ms, _, _, clocks = timed_loop(ctx, w_steps, pg, device, ClockSampler(local), profiled=False)
    mean = reduce_max(pg, statistics.mean(ms), device)
    pms, parts, _, _ = timed_loop(ctx, w_steps, pg, device, None, profiled=True)
    pmean = reduce_max(pg, statistics.mean(pms), device)
    alg = algorithmic(ctx["shape"], ctx["counts"])
    gemm = parts["gemm1_swiglu"] + parts["gemm2_down"]
    T = ctx["shape"][0]
    world = 1 if pg is None else pg.get_world_size()
    out = {"workload": WORKLOAD_NAMES[name], "tokens_per_s": round(T * world / (mean / 1e3), 1),
           "ms_per_step": round(mean, 4), "steps": w_steps,
           # for sub-millisecond steps a few host-side hiccups move the mean
           "ms_per_step_median": round(statistics.median(ms), 4),
           "ms_per_step_max": round(max(ms), 4),
           "kernel_ms": {k_: round(v, 4) for k_, v in parts.items()},
           "ms_per_step_profiled": round(pmean, 4), "expert_rows": ctx["counts"],
           "clocks": clocks, "settle_s": SETTLE_S}
    if name in ("decode", "quarter", "tiny"):
        g_med, g_mean = graph_step_ms(ctx, w_steps)
        g_med = reduce_max(pg, g_med, device)
        out["graph"] = {"ms_per_step_median": round(g_med, 4),
                        "ms_per_step_mean": round(g_mean, 4),
                        "tokens_per_s": round(T * world / (g_med / 1e3), 1),
                        "how": "the same step replayed from a CUDA graph of moe_forward, host "
                               "waiting for each replay (device time without host launch work)"}
    if name == "decode":
        gbs = alg["bytes_experts_decode"] / (gemm / 1000) / 1e9
        out.update({"experts_gbs": round(gbs, 1),
                    "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4),
                    "frac_of_spec_8000": round(gbs / SPEC_HBM_GBS, 4),
                    "layer_gbs": round((alg["bytes_experts_decode"] + alg["bytes_router"]) /
                                       (mean / 1000) / 1e9, 1)})
    else:
        tf = (alg["flops_gemm1"] + alg["flops_gemm2"]) / (gemm / 1000) / 1e12
        out.update({"experts_tflops": round(tf, 1),
                    "frac_of_measured_bf16": round(tf / peaks["bf16_tflops"], 4),
                    "frac_of_spec_2250": round(tf / SPEC_BF16_TFLOPS, 4),
                    "layer_tflops": round(alg["flops_total"] / (mean / 1000) / 1e12, 1)})
    del ctx
    import torch
    torch.cuda.empty_cache()
    return out


def e2e_loop(ctx, steps, warmup, device):
    """The step through the host-I/O entry points, copies inside the timed region.

    queue: one moe_forward_hostio_batches call over the K steps' batches (pinned
    host buffers, four x and four y buffers in rotation): batch b+1's upload and
    batch b-1's download overlap batch b's layer, so only the first upload and
    the last download are exposed; per step = the call's CUDA-event time / K.
    single: one moe_forward_hostio call per step (token chunks inside the call),
    each between two events with the L2 flushed before it.  The host reads every
    batch's result."""
    import torch

    import sparse_mixture_experts_05_b200 as moe
    inp = ctx["inp"]
    shape = ctx["shape"]
    T, d = shape[0], shape[1]
    wargs = (inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    nbuf = 4
    xs = [inp["x"].cpu().pin_memory() for _ in range(nbuf)]
    ys = [torch.empty(T, d, dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    ws = moe.workspace(moe.moe_forward_hostio_batches_workspace_bytes(shape), device)

    def queue(n):
        return ([xs[b % nbuf] for b in range(n)], [ys[b % nbuf] for b in range(n)])

    qx, qy = queue(max(warmup, 2))
    moe.moe_forward_hostio_batches(shape, qx, *wargs, qy, ws)
    torch.cuda.synchronize()
    # like the device-timed steps, which follow only their few warm-up steps: not
    # in the power limiter's response to the profiled pass and warm-up before
    time.sleep(SETTLE_S)
    qx, qy = queue(steps)
    ctx["flush"].fill_(0xA5)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    moe.moe_forward_hostio_batches(shape, qx, *wargs, qy, ws)
    b.record()
    b.synchronize()
    _ = [float(y[0, 0]) for y in ys]  # the host reads the batches' results
    queue_ms = a.elapsed_time(b) / steps
    if moe.moe_read_device_status(ws) != moe.MOE_OK:
        raise RuntimeError("device status error in the end-to-end queue")
    del ws

    ws = moe.workspace(moe.moe_forward_hostio_workspace_bytes(shape), device)
    args = (shape, xs[0], *wargs, ys[0], ws)
    for _ in range(warmup):
        moe.moe_forward_hostio(*args)
    torch.cuda.synchronize()
    ms = []
    for i in range(steps):
        ctx["flush"].fill_(i & 0xFF)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        moe.moe_forward_hostio(*args)
        b.record()
        b.synchronize()
        _ = float(ys[0][0, 0])  # the host reads the step's result
        ms.append(a.elapsed_time(b))
    if moe.moe_read_device_status(ws) != moe.MOE_OK:
        raise RuntimeError("device status error in the end-to-end loop")
    return queue_ms, statistics.mean(ms), T * d * 2, T * d * 2


def router_isolated(ctx, device, launches=60):
    """The router alone: `launches` back-to-back moe_route calls between two
    events, launch i on copy i % n of x, with n copies holding more than twice
    the L2 (so each launch reads its x from DRAM, and nothing dirty is left in
    L2 by a flush).  Reports the per-launch device time against the router's
    algorithmic bytes (x once, W_r, idx and gate)."""
    import torch

    import sparse_mixture_experts_05_b200 as moe
    inp = ctx["inp"]
    shape = ctx["shape"]
    T, d, d_ff, E, k = shape
    x_bytes = T * d * 2
    n = max(2, -(-(256 << 20) // x_bytes))
    xs = [inp["x"].clone() for _ in range(n)]
    idx = torch.empty(T, k, dtype=torch.int32, device=device)
    gate = torch.empty(T, k, dtype=torch.float32, device=device)
    for i in range(2 * n):
        moe.moe_route(shape, xs[i % n], inp["Wg"], inp["bias"], idx=idx, gate=gate)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(launches):
        moe.moe_route(shape, xs[i % n], inp["Wg"], inp["bias"], idx=idx, gate=gate)
    b.record()
    b.synchronize()
    us = a.elapsed_time(b) * 1000.0 / launches
    alg = x_bytes + d * E * 2 + T * k * 8
    peaks, peak_kind = load_peaks()
    gbs = alg / (us * 1e-6) / 1e9
    return {"us_per_launch": round(us, 2), "launches": launches, "x_copies": n,
            "algorithmic_bytes": alg, "achieved_gbs": round(gbs, 1),
            "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "peak_kind": f"{peak_kind} copy bandwidth",
            "note": "back-to-back launches (programmatic overlap between them), each reading "
                    "its own copy of x from DRAM; the step's kernel_ms.router also carries the "
                    "start latency after an event and the write-back of the L2 flush's dirty "
                    "lines that the router's reads evict"}


def oracle_sample(inp, seconds, device_inputs=True):
    """Times the oracle's per-token forward on a sample of tokens; returns dict."""
    import numpy as np

    import oracle
    T, d, d_ff, E, k = inp["shape"]
    host = {key: (inp[key].cpu() if inp[key] is not None else None)
            for key in ("x", "Wg", "bias", "W1", "W3", "W2")}
    oracle.build()
    rng = np.random.default_rng(0)
    t0 = time.perf_counter()
    oracle.forward_tokens(np.array([0], np.int32), host["x"], host["Wg"], host["W1"], host["W3"],
                          host["W2"], k, bias=host["bias"])
    one = max(time.perf_counter() - t0, 1e-4)
    cores = os.cpu_count() or 1
    threads = int(os.environ.get("OMP_NUM_THREADS", cores))
    n = int(max(1, min(T, 4096, seconds / one * min(threads, 64) * 0.8)))
    toks = np.sort(rng.choice(T, n, replace=False)).astype(np.int32)
    t0 = time.perf_counter()
    oracle.forward_tokens(toks, host["x"], host["Wg"], host["W1"], host["W3"], host["W2"], k,
                          bias=host["bias"])
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of the workload's {T} tokens, per-token oracle loop (route, 2 SwiGLU "
                      f"experts, combine) in fp64, {dt:.1f} s wall"}, host


def _omp_threads(n):
    """Sets the OpenMP thread count of this process's runtime (the oracle's)."""
    import ctypes
    try:
        ctypes.CDLL("libgomp.so.1").omp_set_num_threads(int(n))
        return True
    except OSError:
        return False


def oracle_per_config():
    """The oracle's full forward (expert-major loop, fp64) on the tiny,
    quarter-width and decode workloads on all host cores, and on one core (the
    quarter-width and decode ones on a sample through the per-token loop: 64 and
    4 tokens); about 15 s in all.  The prefill and skewed batches are timed on a
    token sample only (`cpu_baseline` itself): their full forward takes minutes."""
    import numpy as np

    import oracle
    from sparse_mixture_experts_05_b200.inputs import workload_inputs
    oracle.build()
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    out = {}
    one_core_sample = {"tiny": None, "quarter": 64, "decode": 4}
    for name in ("tiny", "quarter", "decode"):
        inp = workload_inputs(name)
        T, d, d_ff, E, k = inp["shape"]
        args = (inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], k)
        runs = [("all_cores", cores, None)]
        runs.append(("one_core", 1, one_core_sample[name]))
        for label, threads, sample in runs:
            if not _omp_threads(threads):
                continue
            t0 = time.perf_counter()
            if sample is None:
                oracle.forward(*args)
                n = T
            else:
                toks = np.arange(0, T, T // sample, dtype=np.int32)[:sample]
                oracle.forward_tokens(toks, *args)
                n = len(toks)
            dt = time.perf_counter() - t0
            out[f"{name}_{label}"] = {
                "tokens_per_s": round(n / dt, 2), "threads": threads, "seconds": round(dt, 3),
                "what": ("full forward, expert-major loop" if sample is None else
                         f"{n} of {T} tokens, per-token loop")}
    _omp_threads(cores)
    return out


def run_ours(a):
    import torch

    import sparse_mixture_experts_05_b200 as moe
    world, rank, local, pg = dist_setup(a.gpus)
    torch.cuda.set_device(local)
    device = f"cuda:{local}"
    peaks, peak_kind = load_peaks()
    moe.binding.lib()

    ClockSampler.prepare(local)  # NVML set up before, not inside, the timed region
    ctx = time_workload(a.workload, a.steps, a.warmup, device, rank, a.tokens, a.experts)
    clock = ClockSampler(local)
    step_ms, _, bracket_ms, clocks = timed_loop(ctx, a.steps, pg, device, clock, profiled=False)
    mean_ms = statistics.mean(step_ms)
    max_ms = reduce_max(pg, mean_ms, device)
    # the per-kernel split (and the roofline's kernel time) from a second timed
    # pass of the same steps through moe_forward_profiled
    p_ms, parts, _, _ = timed_loop(ctx, a.steps, pg, device, None, profiled=True)
    p_max_ms = reduce_max(pg, statistics.mean(p_ms), device)
    shape = ctx["shape"]
    T = shape[0]
    alg = algorithmic(shape, ctx["counts"])
    value = T * world / (max_ms / 1000.0)

    e2e_ms, e2e_single_ms, h2d, d2h = e2e_loop(ctx, a.steps, a.warmup, device)
    e2e_ms = reduce_max(pg, e2e_ms, device)
    e2e_single_ms = reduce_max(pg, e2e_single_ms, device)

    gemm_ms = parts["gemm1_swiglu"] + parts["gemm2_down"]
    flops_e = alg["flops_gemm1"] + alg["flops_gemm2"]
    if a.workload in ("decode",):
        achieved = alg["bytes_experts_decode"] / (gemm_ms / 1000) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
                "frac_of_spec_8000": round(achieved / SPEC_HBM_GBS, 4)}
    else:
        achieved = flops_e / (gemm_ms / 1000) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_kind": f"{peak_kind} burst bf16 GEMM",
                "frac_of_sustained": round(achieved / peaks.get("bf16_tflops_sustained", peak), 4),
                "frac_of_spec_2250": round(achieved / SPEC_BF16_TFLOPS, 4)}
    roof["kernel"] = ("expert_gemm_kernel (two launches per step: GEMM1 x.W1|x.W3 -> SiLU(a)*b, "
                      "GEMM2 h.W2); achieved = algorithmic units of both launches / their summed "
                      "CUDA-event time")
    traffic = committed_traffic(a.workload) if a.tokens is None and a.experts is None else None
    roof["traffic"] = traffic
    roof["traffic_scope"] = ("DRAM bytes of both expert_gemm launches of one step, from the committed "
                             "ncu capture of the same kernel source (null once the source changed)")

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(max_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) tokens and N(0,1/fan_in) bf16 weights (no dataset, "
                "no trained weights)",
        "config": {"workload": workload_label(a), "model": "Mixtral 8x7B MoE layer",
                   "T": T, "d": shape[1], "d_ff": shape[2], "E": shape[3], "k": shape[4],
                   "global_batch": T * world, "seq_len": T, "parallelism": f"replicas x{world}",
                   "l2": "flushed: 512 MiB written between timed steps (flush not timed)",
                   "expert_rows": ctx["counts"]},
        "roofline": roof,
        "e2e": {"value": round(T * world / (e2e_ms / 1000.0), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4),
                "api": "moe_forward_hostio_batches: the K steps' batches as one queue (pinned "
                       "host x -> device -> layer -> host y per batch; batch b+1's upload and "
                       "b-1's download overlap batch b's layer); per step = call time / K; "
                       "L2 not flushed between batches (each streams 2.8 GB of expert weights); "
                       "started after its warm-up queue and settle_s idle",
                "settle_s": SETTLE_S,
                "single_call": {"value": round(T * world / (e2e_single_ms / 1000.0), 1),
                                "ms_per_step": round(e2e_single_ms, 4),
                                "api": "moe_forward_hostio once per step (three token chunks "
                                       "inside the call), L2 flushed before each"}},
        "gpu_launches": moe.moe_forward_kernel_count(ctx["shape"]) * a.steps,
        "clocks": clocks,
        "kernel_ms": {k_: round(v, 4) for k_, v in parts.items()},
        "ms_per_step_profiled": round(p_max_ms, 4),
        "timing": ("value and ms_per_step: moe_forward between two CUDA events per step; "
                   "kernel_ms, ms_per_step_profiled and the roofline: a second timed pass of "
                   "the same steps through moe_forward_profiled (events between the launches); "
                   "an event between two launches also takes away their programmatic overlap, "
                   "so each kernel_ms entry includes that kernel's start latency (a few us, "
                   "most visible on the small kernels)"),
        "tflops_layer": round(alg["flops_total"] / (max_ms / 1000) / 1e12, 1),
        "bracket_ms_incl_flush": round(bracket_ms, 3),
    }
    if a.workload in ("prefill", "skew") and not a.no_secondary:
        line["router_isolated"] = router_isolated(ctx, device)
    if a.workload == "prefill" and not a.no_secondary and a.tokens is None and a.experts is None:
        line["extras"] = extras_loop(ctx, a.steps, device, local)
    del ctx
    torch.cuda.empty_cache()

    if a.workload == "prefill" and not a.no_secondary and a.tokens is None and a.experts is None:
        # a decode step is ~0.5 ms: time at least 40 of them so the mean is stable
        line["decode"] = secondary_workload("decode", max(a.steps, 40), a.warmup, device, rank,
                                            local, pg, peaks)
        # the skewed prefill (T = 16384, biased router): ~9 ms a step
        line["skew"] = secondary_workload("skew", min(a.steps, 10), a.warmup, device, rank,
                                          local, pg, peaks)
        # the quarter-width and tiny workloads (~0.1 and ~0.03 ms a step)
        for name in ("quarter", "tiny"):
            line[name] = secondary_workload(name, max(a.steps, 40), a.warmup, device, rank,
                                            local, pg, peaks)

    if world == 1 and rank == 0 and not a.no_cpu_baseline:
        from sparse_mixture_experts_05_b200.inputs import make_inputs
        w = workload(a.workload, a.tokens, a.experts)
        inp = make_inputs(w.T, w.d, w.d_ff, w.E, w.k, w.seed, bias=w.skew_bias, device=device)
        cb, _ = oracle_sample(inp, a.cpu_seconds)
        if a.workload == "prefill" and not a.no_secondary:
            cb["per_config"] = oracle_per_config()
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


# ---------------------------------------------------------------- reference arm (CPU oracle)
def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    import numpy as np

    import oracle
    from sparse_mixture_experts_05_b200.inputs import make_inputs
    w = workload(a.workload, a.tokens, a.experts)
    device = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w.T, w.d, w.d_ff, w.E, w.k, w.seed, bias=w.skew_bias, device=device)
    host = {key: (inp[key].cpu() if inp[key] is not None else None)
            for key in ("x", "Wg", "bias", "W1", "W3", "W2")}
    oracle.build()
    T, k = w.T, w.k
    t0 = time.perf_counter()
    oracle.forward_tokens(np.array([0], np.int32), host["x"], host["Wg"], host["W1"], host["W3"],
                          host["W2"], k, bias=host["bias"])
    one = max(time.perf_counter() - t0, 1e-4)
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    budget = 150.0 / (a.steps + a.warmup)  # whole run within a few minutes
    n = int(max(1, min(T, budget / one * min(threads, 64) * 0.7)))
    rng = np.random.default_rng(1)
    times = []
    for i in range(a.warmup + a.steps):
        toks = np.sort(rng.choice(T, n, replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        oracle.forward_tokens(toks, host["x"], host["Wg"], host["W1"], host["W3"], host["W2"], k,
                              bias=host["bias"])
        if i >= a.warmup:
            times.append(time.perf_counter() - t0)
    step_s = statistics.mean(times)
    value = n / step_s
    sample = (f"{n} random tokens of the workload's {T} per step, per-token oracle loop in fp64 "
              f"(route, k SwiGLU experts, combine)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(step_s * 1000, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same recipe and seeds)",
        "config": {"workload": workload_label(a), "model": "Mixtral 8x7B MoE layer",
                   "T": T, "d": w.d, "d_ff": w.d_ff, "E": w.E, "k": w.k,
                   "global_batch": T, "seq_len": T, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def vs_cublas(a):
    """The expert GEMMs (one moe_expert_swiglu call: GEMM1 with the SwiGLU epilogue,
    then GEMM2) against cuBLAS batched bf16 GEMMs of the same shapes through torch
    (x [E, R/E, d] . [W1|W3] [E, d, 2 d_ff], then h [E, R/E, d_ff] . W2 [E, d_ff, d]),
    with R/E rows per expert so neither side pads.  The two alternate step by step
    with the L2 flushed before each, so both see the same clocks and power state.
    cuBLAS writes bf16 outputs and has no SwiGLU; the comparison is of the
    contractions' throughput."""
    import torch

    import sparse_mixture_experts_05_b200 as moe
    from sparse_mixture_experts_05_b200.inputs import make_inputs

    device = torch.device("cuda", 0)
    w = workload(a.workload, a.tokens, a.experts)
    T, d, d_ff, E, k = w.T, w.d, w.d_ff, w.E, w.k
    R = T * k
    if R % E:
        raise SystemExit("--vs-cublas needs T*k divisible by E")
    inp = make_inputs(R, d, d_ff, E, 1, w.seed, device=device)
    xs = inp["x"]  # used directly as the expert-sorted rows, R/E per expert
    W1, W3, W2 = inp["W1"], inp["W3"], inp["W2"]
    W13 = torch.cat([W1, W3], dim=2).contiguous()
    off = torch.arange(0, R + 1, R // E, dtype=torch.int32, device=device)
    shape = (T, d, d_ff, E, k)
    h = torch.empty(R, d_ff, dtype=torch.bfloat16, device=device)
    o = torch.empty(R, d, dtype=torch.float32, device=device)
    ws = moe.workspace(moe.moe_expert_workspace_bytes(shape), device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    xb = xs.view(E, R // E, d)
    hb = h.view(E, R // E, d_ff)

    def ours():
        moe.moe_expert_swiglu(shape, xs, off, W1, W3, W2, h=h, o=o, ws=ws)

    def cublas():
        torch.bmm(xb, W13)
        torch.bmm(hb, W2)

    for _ in range(a.warmup):
        ours()
        cublas()
    torch.cuda.synchronize()
    times = {"ours": [], "cublas": []}
    clock = ClockSampler(0)
    clock.start()
    for i in range(a.steps):
        for name, fn in (("ours", ours), ("cublas", cublas)):
            flush.fill_(i & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            times[name].append(e0.elapsed_time(e1))
    clocks = clock.stop()
    if moe.moe_read_device_status(ws) != moe.MOE_OK:
        raise RuntimeError("device status error")
    flops = 2.0 * R * d * 2 * d_ff + 2.0 * R * d_ff * d
    med = {n: statistics.median(v) for n, v in times.items()}
    print(json.dumps({
        "metric": "expert GEMM TFLOP/s vs cuBLAS batched bf16 GEMMs (same shapes, alternating)",
        "config": {"workload": workload_label(a), "rows_per_expert": R // E, "d": d,
                   "d_ff": d_ff, "E": E},
        "steps": a.steps, "warmup": a.warmup,
        "ours_ms": round(med["ours"], 4), "cublas_ms": round(med["cublas"], 4),
        "ours_tflops": round(flops / (med["ours"] / 1e3) / 1e12, 1),
        "cublas_tflops": round(flops / (med["cublas"] / 1e3) / 1e12, 1),
        "ours_over_cublas": round(med["cublas"] / med["ours"], 4),
        "ours_ms_all": [round(t, 4) for t in times["ours"]],
        "cublas_ms_all": [round(t, 4) for t in times["cublas"]],
        "clocks": clocks}))


def block_vs_plain(a):
    """The block forward and the plain layer on the block's normalised rows u,
    alternating step by step on the workload's batch (L2 flushed before each
    call), W warm-up pairs then K timed pairs; prints one JSON line of the
    per-call CUDA-event times.  Same routing and GEMM tiles on both sides, so
    the difference is the block edges' cost."""
    import torch

    import sparse_mixture_experts_05_b200 as moe
    device = "cuda:0"
    torch.cuda.set_device(0)
    ctx = time_workload(a.workload, 1, 3, device, 0, a.tokens, a.experts)
    inp = ctx["inp"]
    shape = ctx["shape"]
    T, d = shape[0], shape[1]
    x, Wg, bias, W1, W3, W2 = (inp[key] for key in ("x", "Wg", "bias", "W1", "W3", "W2"))
    gen = torch.Generator(device=device)
    gen.manual_seed(5)
    gamma = (1 + 0.2 * torch.randn(d, generator=gen, device=device)).to(torch.bfloat16)
    ws_b = moe.workspace(moe.moe_block_workspace_bytes(shape), device)
    H = torch.empty(T, d, dtype=torch.bfloat16, device=device)
    moe.moe_block_forward(shape, x, gamma, Wg, bias, W1, W3, W2, H=H, ws=ws_b)
    off = moe.moe_forward_workspace_bytes(shape)
    u = ws_b[off:off + T * d * 2].view(torch.bfloat16).view(T, d).clone()
    calls = {"plain_on_u_ms": lambda: moe.moe_forward(shape, u, Wg, bias, W1, W3, W2,
                                                      y=ctx["y"], ws=ctx["ws"]),
             "block_forward_ms": lambda: moe.moe_block_forward(shape, x, gamma, Wg, bias, W1, W3,
                                                               W2, H=H, ws=ws_b)}
    times = {name: [] for name in calls}
    for i in range(a.warmup + a.steps):
        for name, call in calls.items():
            ctx["flush"].fill_(i & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            e1.synchronize()
            if i >= a.warmup:
                times[name].append(e0.elapsed_time(e1))
    if moe.moe_read_device_status(ws_b) != moe.MOE_OK:
        raise RuntimeError("device status error in the block forward")
    print(json.dumps({"workload": WORKLOAD_NAMES[a.workload], "steps": a.steps,
                      **{name: [round(t, 4) for t in v] for name, v in times.items()}}))


def main(argv=None):
    a = parse(argv)
    if a.impl == "reference":
        run_reference(a)
    elif a.vs_cublas:
        vs_cublas(a)
    elif a.block_vs_plain:
        block_vs_plain(a)
    else:
        run_ours(a)
    return 0


if __name__ == "__main__":
    sys.exit(main())
