"""Benchmark of the W2A8 (ternary i2_s x int8 absmax) linear layer on B200.

Default workload (one step): the decode linears of a BitNet-b1.58-2B-shaped
model at batch 1 -- 30 layers x {QKV 3840x2560, O 2560x2560, gate+up
13824x2560, down 2560x6912}, each with its own seeded weights and input.
A step is one bitnet_w2a8_linear_seq call over the 120 linears (each
quantises its own fp32 x to int8 q, s and computes its fp32 y; one kernel).
Steps run back to back from CUDA graphs of STEPS_PER_GRAPH calls (the
remainder from a one-call graph), so each call's prologue and first weight
copies overlap the previous call's tail through programmatic dependent launch,
as consecutive calls in a stream do; the 520 MB of packed weights exceed the
126 MB L2, so every step streams them from HBM.  Per-linear calls
(bitnet_w2a8_linear) and a dependent chain are timed the same way and
reported beside it.

Metric: achieved HBM GB/s = algorithmic bytes of a step / device time (higher
is better).  Algorithmic bytes per linear: packed codes out*K/4 + one fp32
scale per row (uniform per-tensor absmean scale) + x (4K) + y (4*out); the
two-call path adds the q (K) and s (4) round trip and the GEMV alone counts
codes + row scales + q + s + y.

Also reported in the same JSON line: per-shape GEMV microseconds and GB/s
(L2 flushed before each timed pass), the prefill GEMM int8 TOPS
(T=2048 x {13824x2560, 2560x6912}), the roofline of the dominant kernel, the
oracle timed on the host cores (cpu_baseline), an end-to-end figure with the
inputs copied from pinned host memory and the outputs copied back inside the
timed region (e2e), and SM clocks sampled while timing.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) every rank runs the same workload on its own GPU
(replicas; no data-path collective); value = all ranks' bytes / max time.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W2A8 GEMV µs & achieved HBM GB/s per shape (bs=1); prefill int8 TOPS"
WORKLOAD = "bitnet-b1.58-2B decode linears, batch 1, 30 layers"
LAYERS = 30
STEPS_PER_GRAPH = 10
SHAPES = [("qkv", 3840, 2560), ("o", 2560, 2560), ("gate_up", 13824, 2560), ("down", 2560, 6912)]
PREFILL = [("gate_up", 13824, 2560), ("down", 2560, 6912)]
PREFILL_T = 2048
CONFIG_ID = 1


def step_bytes(shapes=SHAPES, layers=LAYERS, B=1):
    """Algorithmic bytes of one step: (GEMV bytes, act-quant bytes)."""
    gemv = sum(o * k // 4 + 4 * o + B * k + 4 * B + 4 * B * o for _, o, k in shapes) * layers
    quant = sum(4 * B * k + B * k + 4 * B for _, _, k in shapes) * layers
    return gemv, quant


def gemv_bytes(out, K, B=1):
    return out * K // 4 + 4 * out + B * K + 4 * B + 4 * B * out


def linear_bytes(out, K, B=1):
    """Fused path: packed codes + row scales + fp32 x in + fp32 y out."""
    return out * K // 4 + 4 * out + 4 * B * K + 4 * B * out


def fused_step_bytes(shapes=SHAPES, layers=LAYERS, B=1):
    return sum(linear_bytes(o, k, B) for _, o, k in shapes) * layers


def reduce_max(values, device):
    """Element-wise max over all ranks (torch.distributed), e.g. of per-rank
    device times; identity on a single process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate(per_rank_ms, per_rank_bytes):
    """Whole-job throughput: all ranks' bytes over the slowest rank's time (GB/s)."""
    t = max(per_rank_ms)
    return sum(per_rank_bytes) / (t * 1e-3) / 1e9, t


# --------------------------------------------------------------- clocks --

class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled every 100 ms
    through NVML (read-only queries) while the timed region runs.  The device is
    found by its UUID, so the index under CUDA_VISIBLE_DEVICES does not matter.
    Falls back to `nvidia-smi -lms` with line-buffered output if NVML cannot be
    loaded (a fully buffered pipe loses every sample when the tool is stopped)."""

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("hw_power_brake_slowdown", 0x80), ("sw_power_cap", 0x4))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active")

    def __init__(self, device):
        self.device = device
        self.samples = []  # (time, sm_mhz, max_mhz, power_w, reasons bitmask)
        self.t0 = self.t1 = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        self.source = "none"

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except pynvml.NVMLError:
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.source = "nvml"

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append((time.time(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), mx,
                                             nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                             nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                    except nv.NVMLError:
                        pass
                    self._stop.wait(0.1)
            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
            return
        except Exception:
            pass
        try:
            import torch
            idx = str(torch.cuda.get_device_properties(self.device).uuid)
            self._proc = subprocess.Popen(
                ["stdbuf", "-oL", "nvidia-smi", "-i", "GPU-" + idx, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"

            def read():
                for line in self._proc.stdout:
                    p = [x.strip() for x in line.split(",")]
                    try:
                        self.samples.append((time.time(), float(p[0]), float(p[1]), float(p[2]), int(p[3], 16)))
                    except (ValueError, IndexError):
                        continue
            self._thread = threading.Thread(target=read, daemon=True)
            self._thread.start()
        except (OSError, RuntimeError):
            self._proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        self._stop.set()
        if self._proc:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread:
            self._thread.join(timeout=2)

    def summary(self):
        rows = [r for r in self.samples if self.t0 is None or (self.t0 <= r[0] <= (self.t1 or r[0]))]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0,
                    "source": self.source}
        mhz = sorted(r[1] for r in rows)
        reasons = sorted({n for r in rows for n, bit in self.REASONS if r[4] & bit})
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_min_mhz": mhz[0], "sm_max_mhz": rows[-1][2],
                "power_w_median": sorted(r[3] for r in rows)[len(rows) // 2], "reasons": reasons,
                "samples": len(rows), "source": self.source}


# ----------------------------------------------------------- our arm --

def build_weights(b, torch, dev, layers, shapes, config):
    """Seeded fp32 N(0,1) weights (the splitmix64 + Box-Muller stream of
    synthetic/, drawn on the device), ternarised with per-tensor absmean and
    packed by the library, then repacked.  Untimed setup."""
    import synthetic as syn
    ws = {}
    maxn = max(o * k for _, o, k in shapes)
    maxo, maxk = max(o for _, o, _ in shapes), max(k for _, _, k in shapes)
    cbuf = torch.empty(maxn // 4, dtype=torch.uint8, device=dev)
    sbuf = torch.empty(maxn // 128, dtype=torch.float32, device=dev)
    wsp = torch.empty(b.bitnet_ternarize_workspace_bytes(maxo, maxk) + 4096, dtype=torch.uint8, device=dev)
    for l in range(layers):
        for m, (name, o, k) in enumerate(shapes):
            w = syn.normal_device(syn.seed_for(config, l, m, syn.KIND_WEIGHT), o * k, dev)
            b.bitnet_ternarize_absmean_device(w, o, k, b.BITNET_ABSMEAN_PER_TENSOR, cbuf[:o * k // 4],
                                              sbuf[:o * k // 128], wsp)
            data = torch.empty(b.bitnet_repacked_bytes(o, k), dtype=torch.uint8, device=dev)
            ws[(l, name)] = b.bitnet_repack_device(cbuf[:o * k // 4], sbuf[:o * k // 128], o, k, data)
            del w
    del cbuf, sbuf, wsp
    return ws


def make_inputs(torch, dev, layers, shapes, B, config, outliers=True):
    """x for every linear from the host recipe of synthetic/ (N(0,1), a fixed
    1% of channels x20): one flat fp32 device buffer and its pinned host copy."""
    import numpy as np

    import synthetic as syn
    parts, views, off = [], {}, 0
    for l in range(layers):
        for m, (name, o, k) in enumerate(shapes):
            parts.append(syn.activations(syn.seed_for(config, l, m, syn.KIND_ACT), B, k, outliers=outliers,
                                         outlier_seed=syn.seed_for(config, 0, m, syn.KIND_OUTLIER)).reshape(-1))
            views[(l, name)] = (off, B * k)
            off += B * k
    host = torch.from_numpy(np.concatenate(parts)).pin_memory()
    return host, host.to(dev), views


class Timer:
    """CUDA-graph replays timed with CUDA events on the replay stream."""

    def __init__(self, torch, stream, dev):
        self.torch, self.stream, self.dev = torch, stream, dev

    def capture(self, fn, warm=2):
        t = self.torch
        with t.cuda.stream(self.stream):
            for _ in range(warm):
                fn()
        t.cuda.synchronize(self.dev)
        g = t.cuda.CUDAGraph()
        with t.cuda.graph(g, stream=self.stream):
            fn()
        return g

    def ms(self, graph, replays=20, passes=5, pre=None):
        """Median over `passes` of the mean ms per replay (`pre` runs untimed
        before each pass, e.g. an L2 flush)."""
        t = self.torch
        out = []
        for _ in range(passes):
            with t.cuda.stream(self.stream):
                if pre:
                    pre()
                e0, e1 = t.cuda.Event(enable_timing=True), t.cuda.Event(enable_timing=True)
                e0.record(self.stream)
                for _ in range(replays):
                    graph.replay()
                e1.record(self.stream)
            e1.synchronize()
            out.append(e0.elapsed_time(e1) / replays)
        return sorted(out)[len(out) // 2]


def hbm(nbytes, ms, peak):
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"us": round(ms * 1e3, 3), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4)}


def linear_entries(weights, layers, shapes, x_dev, xviews, ys, chain=False):
    """(Weight, x, y, wait_for) for the sequence call: every linear with its own
    x, or (chain) each x the first K outputs of the previous linear's y."""
    ents = []
    for l in range(layers):
        for name, o, k in shapes:
            i = len(ents)
            key = (l, name)
            if chain and i > 0:
                ents.append((weights[key], ys[i - 1][:k], ys[i], i - 1))
            else:
                xo, xn = xviews[key]
                ents.append((weights[key], x_dev[xo:xo + xn], ys[i], -1))
    return ents


def run_ours(args, rank, world, dev):
    import torch

    import ternary_weight_absmax_b200 as b

    torch.cuda.set_device(dev)
    B = 1
    peaks = read_peaks()
    peak = peaks["hbm_gbs"]
    weights = build_weights(b, torch, dev, LAYERS, SHAPES, CONFIG_ID)
    x_host, x_dev, xviews = make_inputs(torch, dev, LAYERS, SHAPES, B, CONFIG_ID)
    ytot = sum(B * o for _, o, _ in SHAPES) * LAYERS
    y_dev = torch.empty(ytot, dtype=torch.float32, device=dev)
    y_host = torch.empty(ytot, dtype=torch.float32).pin_memory()
    ys, off = [], 0
    for l in range(LAYERS):
        for name, o, k in SHAPES:
            ys.append(y_dev[off:off + B * o])
            off += B * o
    n_lin = LAYERS * len(SHAPES)
    stream = torch.cuda.Stream(device=dev)
    T = Timer(torch, stream, dev)
    seq = linear_entries(weights, LAYERS, SHAPES, x_dev, xviews, ys)
    g_step = T.capture(lambda: b.bitnet_w2a8_linear_seq(seq))
    g_steps = T.capture(lambda: [b.bitnet_w2a8_linear_seq(seq) for _ in range(STEPS_PER_GRAPH)])
    launches_per_step = 1

    def run_steps(k):
        """Exactly k steps: k // STEPS_PER_GRAPH replays of the multi-call graph, then one-call replays."""
        for _ in range(k // STEPS_PER_GRAPH):
            g_steps.replay()
        for _ in range(k % STEPS_PER_GRAPH):
            g_step.replay()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    clocks = ClockSampler(dev)
    clocks.start()
    with torch.cuda.stream(stream):
        run_steps(args.warmup)
    barrier()
    # ---- timed region: K steps back to back (the 520 MB of weights exceed L2) ----
    clocks.mark("t0")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        run_steps(args.steps)
        e1.record(stream)
    e1.synchronize()
    barrier()
    clocks.mark("t1")
    step_ms_local = e0.elapsed_time(e1) / args.steps
    clocks.stop()

    # ---- e2e: pinned host x -> device, the C-ABI call, y -> pinned host ----
    # Every step copies its own inputs in and its outputs out, inside the timed
    # region.  Two device buffer sets let step i + 1's inputs copy in (on a
    # copy stream) while step i computes, and step i's outputs copy out on a
    # third stream: the transfers overlap the compute and each other (PCIe is
    # full duplex), as a serving loop would run it.
    x_dev_b = torch.empty_like(x_dev)
    y_dev_b = torch.empty_like(y_dev)
    ys_b, off = [], 0
    for l in range(LAYERS):
        for name, o, k in SHAPES:
            ys_b.append(y_dev_b[off:off + B * o])
            off += B * o
    seq_b = linear_entries(weights, LAYERS, SHAPES, x_dev_b, xviews, ys_b)
    g_step_b = T.capture(lambda: b.bitnet_w2a8_linear_seq(seq_b))
    xs2, ys2, gs2 = [x_dev, x_dev_b], [y_dev, y_dev_b], [g_step, g_step_b]
    y_host2 = [y_host, torch.empty_like(y_host).pin_memory()]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = {n: [torch.cuda.Event(), torch.cuda.Event()] for n in ("in", "comp", "out")}

    def e2e_run(steps):
        for i in range(steps):
            k = i & 1
            if i >= 2:
                s_in.wait_event(ev["comp"][k])       # step i - 2 has read xs2[k]
            with torch.cuda.stream(s_in):
                xs2[k].copy_(x_host, non_blocking=True)
                ev["in"][k].record(s_in)
            stream.wait_event(ev["in"][k])
            if i >= 2:
                stream.wait_event(ev["out"][k])      # step i - 2's outputs left ys2[k]
            with torch.cuda.stream(stream):
                gs2[k].replay()
                ev["comp"][k].record(stream)
            s_out.wait_event(ev["comp"][k])
            with torch.cuda.stream(s_out):
                y_host2[k].copy_(ys2[k], non_blocking=True)
                ev["out"][k].record(s_out)
    e2e_run(4)
    torch.cuda.synchronize(dev)
    e2e_steps = max(4, min(args.steps, 500))
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    stream.wait_event(f0)
    s_out.wait_event(f0)
    e2e_run(e2e_steps)
    s_in.wait_event(ev["out"][(e2e_steps - 1) & 1])
    s_in.wait_event(ev["out"][e2e_steps & 1])
    f1.record(s_in)
    f1.synchronize()
    assert torch.equal(y_host2[0], y_host2[1]), "the two e2e buffer sets disagree"
    e2e_ms_local = f0.elapsed_time(f1) / e2e_steps

    per_rank_bytes = fused_step_bytes()
    side = {}
    # ---- the same step, one bitnet_w2a8_linear call per linear ----
    g_calls = T.capture(lambda: [b.bitnet_w2a8_linear(w, x, 1, y) for (w, x, y, _) in seq])
    side["per_call_step"] = dict(hbm(per_rank_bytes, T.ms(g_calls, 20), peak), launches=n_lin,
                                 how="bitnet_w2a8_linear per linear (batch-1 decode kernel, programmatic "
                                     "dependent launch), 120 calls in one CUDA graph")
    del g_calls
    # ---- dependent chain: each x is the first K outputs of the previous y ----
    chain = linear_entries(weights, LAYERS, SHAPES, x_dev, xviews, ys, chain=True)
    work = torch.zeros(b.bitnet_w2a8_linear_seq_workspace_bytes(n_lin), dtype=torch.uint8, device=dev)
    try:
        g_chain = T.capture(lambda: b.bitnet_w2a8_linear_seq(chain, work))
        g_chain_calls = T.capture(lambda: [b.bitnet_w2a8_linear(w, x, 1, y) for (w, x, y, _) in chain])
        side["chained_step"] = {
            "seq": dict(hbm(per_rank_bytes, T.ms(g_chain, 20), peak), launches=1),
            "per_call": dict(hbm(per_rank_bytes, T.ms(g_chain_calls, 20), peak), launches=n_lin),
            "how": "linear i reads the first K outputs of linear i-1 (QKV->O->gate+up->down->next QKV): one "
                   "bitnet_w2a8_linear_seq call whose entries wait for their producer on the device, vs one "
                   "bitnet_w2a8_linear call per linear"}
        del g_chain, g_chain_calls
    except Exception as e:  # reported beside the headline, never instead of it
        side["chained_step"] = {"error": f"{type(e).__name__}: {e}"}
    del g_step, g_steps
    torch.cuda.synchronize(dev)
    side["per_shape"] = run_per_shape(b, torch, dev, T, weights, peak)
    side["llama8b_sweep"] = run_llama8b(b, torch, dev, T, peaks)
    side["prefill"] = run_prefill(b, torch, dev, T, peaks)
    side["small_batch_gemv"] = run_small_batch(b, torch, dev, T, weights, peak)
    side["block_scale"] = run_block_scale(b, torch, dev, T, peaks)
    side["lut_gemv_b1"] = run_lut(b, torch, dev, T, weights)

    status = b.bitnet_get_device_error(stream.cuda_stream)
    if status != b.BITNET_OK:
        raise RuntimeError(f"device error after bench: {b.bitnet_status_string(status)}")

    step_ms, e2e_ms = reduce_max([step_ms_local, e2e_ms_local], dev)
    value, _ = aggregate([step_ms] * world, [per_rank_bytes] * world)
    e2e_value, _ = aggregate([e2e_ms] * world, [per_rank_bytes] * world)
    # Dominant kernel: decode_seq_kernel, one launch per step; its average
    # launch time is the step time (CUDA events on the launch stream, timed
    # region above).
    launch_us = step_ms * 1e3 / launches_per_step
    bytes_per_launch = per_rank_bytes / launches_per_step
    achieved = bytes_per_launch / (launch_us * 1e-6) / 1e9
    traffic, traffic_note = read_traffic("decode_seq_kernel", bytes_per_launch)
    roofline = {"kernel": "decode_seq_kernel (bitnet_w2a8_linear_seq, 120 batch-1 linears per launch)",
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": peaks["source"], "traffic": traffic,
                "traffic_source": traffic_note, "bytes_per_launch": round(bytes_per_launch, 1),
                "launch_us": round(launch_us, 3)}

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (splitmix64 + Box-Muller N(0,1) weights, per-tensor absmean ternary; N(0,1) "
                "activations with 1% of channels x20)",
        "path": "bitnet_w2a8_linear_seq: one call per step over the 120 linears, each quantising its own "
                "fp32 x (absmax int8) and computing its fp32 y",
        "config": {"workload": WORKLOAD, "shapes_out_x_K": [[o, k] for _, o, k in SHAPES], "layers": LAYERS,
                   "batch": B, "linears_per_step": n_lin,
                   "inputs": "every linear has its own seeded input (the linears of the step do not depend on "
                             "each other); chained_step reports the dependent variant",
                   "l2": "inputs larger than L2 (520 MB packed weights per step, read once per step)",
                   "graph": f"CUDA graphs of {STEPS_PER_GRAPH} step calls replayed back to back (remainder: a "
                            "one-call graph); programmatic dependent launch between calls",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        **side,
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": int(x_host.numel() * 4), "d2h_bytes_per_step": int(y_host.numel() * 4),
                "how": "per step: pinned x copied in, the step's C-ABI call (graph), y copied out to pinned memory; "
                       "two buffer sets, so the next step's copy in and this step's copy out overlap the compute"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    return out


def run_per_shape(b, torch, dev, T, weights, peak):
    """Per shape of the step: (a) one bitnet_w2a8_linear call (latency of an
    isolated launch: 30 calls on the 30 layers' weights in a graph, each with
    its own cold x, L2 flushed before each pass), (b) sustained: the 30 layers'
    weights of that shape in one bitnet_w2a8_linear_seq call."""
    res = {}
    try:
        flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        for m, (name, o, k) in enumerate(SHAPES):
            ws = [weights[(l, name)] for l in range(LAYERS)]
            xs = [torch.randn(k, device=dev) for _ in range(LAYERS)]
            ys = [torch.empty(o, device=dev) for _ in range(LAYERS)]
            g1 = T.capture(lambda: [b.bitnet_w2a8_linear(w, x, 1, y) for w, x, y in zip(ws, xs, ys)])
            g2 = T.capture(lambda: b.bitnet_w2a8_linear_seq([(w, x, y, -1) for w, x, y in zip(ws, xs, ys)]))
            one = T.ms(g1, 1, 7, pre=lambda: flush.fill_(1.0)) / LAYERS
            sus = T.ms(g2, 1, 7, pre=lambda: flush.fill_(1.0)) / LAYERS
            nb = linear_bytes(o, k)
            res[name] = {"out": o, "K": k, "bytes": nb, "per_call": hbm(nb, one, peak),
                         "sustained_seq": hbm(nb, sus, peak)}
            del g1, g2
        del flush
    except Exception as e:
        res["error"] = f"{type(e).__name__}: {e}"
    return res


SHAPES_8B = [("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_up", 28672, 4096), ("down", 4096, 14336)]
LAYERS_8B = 32
CONFIG_8B = 4


def run_llama8b(b, torch, dev, T, peaks):
    """Llama-3-8B-shaped ternary linears, 32 layers (1.97 GB packed): the
    sustained-HBM sweep at batch 1 (independent inputs and the dependent
    chain), at batch 16 and as prefill (T = 1024)."""
    peak = peaks["hbm_gbs"]
    res = {"shapes_out_x_K": [[o, k] for _, o, k in SHAPES_8B], "layers": LAYERS_8B}
    try:
        weights = build_weights(b, torch, dev, LAYERS_8B, SHAPES_8B, CONFIG_8B)
        packed = sum(weights[key].rows * weights[key].cols // 4 for key in weights)
        res["packed_bytes"] = packed
        n_lin = LAYERS_8B * len(SHAPES_8B)
        for B in (1, 16):
            x_host, x_dev, xviews = make_inputs(torch, dev, LAYERS_8B, SHAPES_8B, B, CONFIG_8B)
            ytot = sum(B * o for _, o, _ in SHAPES_8B) * LAYERS_8B
            y_dev = torch.empty(ytot, dtype=torch.float32, device=dev)
            ys, off = [], 0
            for l in range(LAYERS_8B):
                for name, o, k in SHAPES_8B:
                    ys.append(y_dev[off:off + B * o])
                    off += B * o
            nbytes = fused_step_bytes(SHAPES_8B, LAYERS_8B, B)
            if B == 1:
                seq = linear_entries(weights, LAYERS_8B, SHAPES_8B, x_dev, xviews, ys)
                g = T.capture(lambda: b.bitnet_w2a8_linear_seq(seq))
                res["b1_seq"] = dict(hbm(nbytes, T.ms(g, 10), peak), launches=1)
                del g
                g = T.capture(lambda: [b.bitnet_w2a8_linear(w, x, 1, y) for (w, x, y, _) in seq])
                res["b1_per_call"] = dict(hbm(nbytes, T.ms(g, 10), peak), launches=n_lin)
                del g
                chain = linear_entries(weights, LAYERS_8B, SHAPES_8B, x_dev, xviews, ys, chain=True)
                work = torch.zeros(b.bitnet_w2a8_linear_seq_workspace_bytes(n_lin), dtype=torch.uint8, device=dev)
                try:
                    g = T.capture(lambda: b.bitnet_w2a8_linear_seq(chain, work))
                    res["b1_chain_seq"] = dict(hbm(nbytes, T.ms(g, 10), peak), launches=1)
                    del g
                except Exception as e:
                    res["b1_chain_seq"] = {"error": f"{type(e).__name__}: {e}"}
            else:
                ents = linear_entries(weights, LAYERS_8B, SHAPES_8B, x_dev, xviews, ys)
                maxk = max(k for _, _, k in SHAPES_8B)
                qb = torch.empty(B * maxk, dtype=torch.int8, device=dev)
                sb = torch.empty(B, dtype=torch.float32, device=dev)
                g = T.capture(lambda: [b.bitnet_w2a8_linear(w, x, B, y, qb[:B * w.cols], sb)
                                       for (w, x, y, _) in ents])
                res[f"b{B}_per_call"] = dict(hbm(nbytes, T.ms(g, 5), peak), launches=2 * n_lin,
                                             how="bitnet_w2a8_linear per linear with q_out / s_out: the "
                                                 "quantiser, then the tensor-core GEMV")
                del g
            del x_host, x_dev, y_dev, ys
        # Prefill T = 1024: act-quant + GEMM per shape (layer 0's weights).
        res["prefill_T1024"] = prefill_shapes(b, torch, dev, T, peaks, [(n, o, k, weights[(0, n)])
                                                                        for n, o, k in SHAPES_8B], 1024)
        del weights
        torch.cuda.empty_cache()
    except Exception as e:
        res["error"] = f"{type(e).__name__}: {e}"
    return res


def prefill_shapes(b, torch, dev, T, peaks, cases, tokens):
    """Per shape: bitnet_w2a8_gemm (weights decoded in the kernel, per
    128-token tile), bitnet_w2a8_gemm_ws (weights expanded to int8 once per
    call, then the pair-of-SMs GEMM), the quantiser, the quantiser followed
    by bitnet_w2a8_gemm (linear_us), and bitnet_w2a8_linear_ws (linear_ws_us:
    one kernel quantises x and expands the weights, then the pair GEMM)."""
    out = {}
    for name, o, k, w in cases:
        x = torch.randn(tokens * k, dtype=torch.float32, device=dev)
        q = torch.empty(tokens * k, dtype=torch.int8, device=dev)
        s = torch.empty(tokens, dtype=torch.float32, device=dev)
        y = torch.empty(tokens * o, dtype=torch.float32, device=dev)
        ws = torch.empty(b.bitnet_w2a8_gemm_workspace_bytes(o, k), dtype=torch.uint8, device=dev)
        g_q = T.capture(lambda: b.bitnet_quant_act(x, tokens, k, q, s))
        g_m = T.capture(lambda: b.bitnet_w2a8_gemm(w, q, s, tokens, y))
        g_w = T.capture(lambda: b.bitnet_w2a8_gemm_ws(w, q, s, tokens, y, ws))
        g_b = T.capture(lambda: (b.bitnet_quant_act(x, tokens, k, q, s), b.bitnet_w2a8_gemm(w, q, s, tokens, y)))
        g_bw = T.capture(lambda: b.bitnet_w2a8_linear_ws(w, x, tokens, y, q, s, ws))
        mq, mm, mw, mb, mbw = T.ms(g_q, 10), T.ms(g_m, 10), T.ms(g_w, 10), T.ms(g_b, 10), T.ms(g_bw, 10)
        ops = 2.0 * tokens * o * k
        tops = ops / (mm * 1e-3) / 1e12
        tops_w = ops / (mw * 1e-3) / 1e12
        qbytes = 4 * tokens * k + tokens * k + 4 * tokens
        out[name] = {"out": o, "K": k, "T": tokens, "gemm_us": round(mm * 1e3, 2), "TOPS": round(tops, 1),
                     "frac_of_int8_peak": round(tops / peaks["int8_tops"], 4),
                     "gemm_ws_us": round(mw * 1e3, 2), "ws_TOPS": round(tops_w, 1),
                     "ws_frac_of_int8_peak": round(tops_w / peaks["int8_tops"], 4),
                     "act_quant_us": round(mq * 1e3, 2),
                     "act_quant_GB/s": round(qbytes / (mq * 1e-3) / 1e9, 1),
                     "linear_us": round(mb * 1e3, 2), "linear_ws_us": round(mbw * 1e3, 2)}
        del g_q, g_m, g_w, g_b, g_bw, ws
    return out


def run_prefill(b, torch, dev, T, peaks):
    res = {"int8_peak_TOPS": peaks["int8_tops"], "peak_source": peaks["int8_source"]}
    try:
        weights = build_weights(b, torch, dev, 1, PREFILL, 3)
        for tokens in (512, 2048):
            res[f"T{tokens}"] = prefill_shapes(b, torch, dev, T, peaks,
                                               [(n, o, k, weights[(0, n)]) for n, o, k in PREFILL], tokens)
        best = max(max(v["TOPS"], v["ws_TOPS"]) for tt in ("T512", "T2048") for v in res[tt].values())
        res["best_frac_of_int8_peak"] = round(best / peaks["int8_tops"], 4)
        del weights
    except Exception as e:  # reported beside the headline, never instead of it
        res["error"] = f"{type(e).__name__}: {e}"
    return res


SMALL_BATCH = [("o", 2560, 2560), ("gate_up", 13824, 2560), ("wide", 20480, 3200)]
SMALL_BATCH_B = (1, 4, 16)


def run_small_batch(b, torch, dev, T, weights, peak):
    """bitnet_w2a8_gemv at B = 1, 4, 16 on the standalone shapes: one call per
    distinct weight copy (30 copies of the step's O and gate+up weights, 12
    copies of 20480 x 3200), one q shared by the calls, L2 flushed with a
    512 MB write before each timed pass; median of 5 passes, us per call and
    algorithmic GB/s."""
    res = {}
    try:
        wide = build_weights(b, torch, dev, 12, [("wide", 20480, 3200)], 2)
        flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        for name, o, k in SMALL_BATCH:
            ws = [wide[(l, name)] for l in range(12)] if name == "wide" else \
                [weights[(l, name)] for l in range(LAYERS)]
            res[name] = {"out": o, "K": k}
            for B in SMALL_BATCH_B:
                x = torch.randn(B * k, dtype=torch.float32, device=dev)
                q = torch.empty(B * k, dtype=torch.int8, device=dev)
                s = torch.empty(B, dtype=torch.float32, device=dev)
                y = torch.empty(B * o, dtype=torch.float32, device=dev)
                b.bitnet_quant_act(x, B, k, q, s)
                g = T.capture(lambda: [b.bitnet_w2a8_gemv(w, q, s, B, y) for w in ws])
                ms = T.ms(g, 1, 5, pre=lambda: flush.fill_(1.0)) / len(ws)
                res[name][f"B{B}"] = hbm(gemv_bytes(o, k, B), ms, peak)
                del g
        del flush, wide
    except Exception as e:  # reported beside the headline, never instead of it
        res["error"] = f"{type(e).__name__}: {e}"
    return res


def run_block_scale(b, torch, dev, T, peaks):
    """The general (per-block scale) paths on varied scales: every 128-weight
    block with its own absmean scale (the library's per-block ternariser).
    GEMV B = 1 (general kernel, fp64 epilogue) over 30 copies of 13824 x 2560
    with L2 flushed, and the GEMM at T = 2048 (block-scale tcgen05 path)."""
    res = {}
    try:
        import synthetic as syn
        o, k = 13824, 2560
        cbuf = torch.empty(o * k // 4, dtype=torch.uint8, device=dev)
        sbuf = torch.empty(o * k // 128, dtype=torch.float32, device=dev)
        wsp = torch.empty(b.bitnet_ternarize_workspace_bytes(o, k) + 4096, dtype=torch.uint8, device=dev)
        ws = []
        for l in range(30):
            w = syn.normal_device(syn.seed_for(5, l, 0, syn.KIND_WEIGHT), o * k, dev)
            b.bitnet_ternarize_absmean_device(w, o, k, b.BITNET_ABSMEAN_PER_BLOCK, cbuf, sbuf, wsp)
            data = torch.empty(b.bitnet_repacked_bytes(o, k), dtype=torch.uint8, device=dev)
            ws.append(b.bitnet_repack_device(cbuf, sbuf, o, k, data))
            assert not ws[-1].uniform
        flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        x = torch.randn(k, device=dev)
        q = torch.empty(k, dtype=torch.int8, device=dev)
        s = torch.empty(1, device=dev)
        y = torch.empty(o, device=dev)
        b.bitnet_quant_act(x, 1, k, q, s)
        g = T.capture(lambda: [b.bitnet_w2a8_gemv(w, q, s, 1, y) for w in ws])
        ms = T.ms(g, 1, 5, pre=lambda: flush.fill_(1.0)) / len(ws)
        nb = o * k // 4 + o * k // 32 + k + 4 + 4 * o
        res["gemv_b1_13824x2560"] = dict(hbm(nb, ms, peaks["hbm_gbs"]), bytes=nb,
                                         how="bitnet_w2a8_gemv, general kernel (block scales, fp64 epilogue)")
        del g, flush
        res["gemm_T2048_13824x2560"] = prefill_shapes(b, torch, dev, T, peaks, [("gate_up", o, k, ws[0])], 2048)[
            "gate_up"]
        del ws, cbuf, sbuf, wsp
    except Exception as e:
        res["error"] = f"{type(e).__name__}: {e}"
    return res


def run_lut(b, torch, dev, T, weights):
    """The table-lookup GEMV variant against the dp4a GEMV at batch 1 on the
    step's four shapes: 30 calls on the 30 layers' weights, one q, L2 flushed
    before each timed pass, median of 5 passes, us per call."""
    res = {}
    try:
        flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        for name, o, k in SHAPES:
            ws = [weights[(l, name)] for l in range(LAYERS)]
            x = torch.randn(k, dtype=torch.float32, device=dev)
            q = torch.empty(k, dtype=torch.int8, device=dev)
            s = torch.empty(1, dtype=torch.float32, device=dev)
            y = torch.empty(o, dtype=torch.float32, device=dev)
            b.bitnet_quant_act(x, 1, k, q, s)
            res[name] = {"out": o, "K": k}
            for kind, call in (("lut", lambda w: b.bitnet_w2a8_gemv_lut(w, q, s, y)),
                               ("dp4a", lambda w: b.bitnet_w2a8_gemv(w, q, s, 1, y))):
                g = T.capture(lambda: [call(w) for w in ws])
                res[name][f"{kind}_us"] = round(T.ms(g, 1, 5, pre=lambda: flush.fill_(1.0)) / len(ws) * 1e3, 3)
                del g
        del flush
    except Exception as e:  # reported beside the headline, never instead of it
        res["error"] = f"{type(e).__name__}: {e}"
    return res


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        hbm_, bf16 = float(d["hbm_gbs"]), float(d["bf16_tflops"])
        src = "measured (MEASURED_PEAKS.json: copy bandwidth)"
        isrc = "measured bf16 cuBLAS burst x 2 (nominal int8:bf16 dense ratio)"
    except (OSError, KeyError, ValueError):
        hbm_, bf16 = 6650.0, 1590.0
        src = isrc = "fallback (6.65 TB/s, 1.59 PFLOP/s bf16; no MEASURED_PEAKS.json)"
    return {"hbm_gbs": hbm_, "int8_tops": 2.0 * bf16, "source": src, "int8_source": isrc}


def source_digest(*names):
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "ternary_weight_absmax_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic(kernel, bytes_per_launch):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    summary, scaled to this launch's algorithmic bytes when the capture ran a
    smaller case; null if the kernel's source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)[kernel]
    except (OSError, ValueError, KeyError):
        return None, "no ncu capture on record"
    if d.get("source_digest") != source_digest(*d.get("sources", [])):
        return None, "kernel changed since the ncu capture"
    ratio = bytes_per_launch / d["algorithmic_bytes"]
    note = f"ncu dram__bytes_read.sum + dram__bytes_write.sum, {d['case']}"
    if abs(ratio - 1.0) > 1e-6:
        note += f", scaled x{ratio:.4f} to this launch's algorithmic bytes"
    return round(d["dram_bytes"] * ratio), note


# ----------------------------------------------------- reference arm --

def run_reference(args, rank, world):
    """The oracle (plain C, one host core) on a bounded sample of the same
    workload: a seeded slice of output rows of each of the four linears of
    layer 0, sized so the whole run stays within a few minutes."""
    import numpy as np

    import oracle
    import synthetic as syn

    oracle.build()
    B = 1
    budget_s = float(os.environ.get("BENCH_REFERENCE_BUDGET_S", "60"))
    nsteps = args.steps + args.warmup
    per_step = max(budget_s / max(nsteps, 1), 0.002)
    # Calibrate: rows per step so one step takes about per_step seconds.
    cases = []
    for m, (name, o, k) in enumerate(SHAPES):
        rows = 64
        w = syn.normal_matrix(syn.seed_for(CONFIG_ID, 0, m, syn.KIND_WEIGHT), rows, k)
        t, g = oracle.absmean_tensor(w)
        codes = oracle.pack_i2s(t)
        sc = np.full((rows, k // 128), g, dtype=np.float32)
        x = syn.activations(syn.seed_for(CONFIG_ID, 0, m, syn.KIND_ACT), B, k, outliers=True)
        cases.append((name, k, codes, sc, x))

    def one(frac_rows):
        nbytes = 0
        for name, k, codes, sc, x in cases:
            r = max(1, int(frac_rows))
            q, s, _ = oracle.quant_act(x)
            oracle.linear(codes[:r], sc[:r], k, q, s)
            nbytes += linear_bytes(r, k)
        return nbytes

    t0 = time.perf_counter()
    one(64)
    dt64 = time.perf_counter() - t0
    rows = int(max(1, min(64, 64 * per_step / max(dt64, 1e-9))))
    for _ in range(args.warmup):
        one(rows)
    t0 = time.perf_counter()
    total = 0
    for _ in range(args.steps):
        total += one(rows)
    dt = time.perf_counter() - t0
    value = total / dt / 1e9
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / max(args.steps, 1), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded)", "config": {"workload": WORKLOAD, "batch": B, "layers_sampled": 1,
                                                  "rows_per_linear_per_step": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{rows} output rows of each of the 4 linears of layer 0 per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return out


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(seconds=8.0):
    """The oracle (plain single-threaded C) timed on the host on a bounded
    sample of the workload: layer 0's four linears (all rows, batch 1), (a) on
    one core, (b) split by output rows over one thread per host core (the C
    call releases the GIL), each for about `seconds`; plus the prefill GEMM
    oracle on a 64-token slice of 13824 x 2560, all cores, extrapolated
    linearly to T = 2048."""
    import concurrent.futures as cf

    import numpy as np

    import oracle
    import synthetic as syn

    oracle.build()
    cores = os.cpu_count() or 1
    cases = []
    for m, (name, o, k) in enumerate(SHAPES):
        w = syn.normal_matrix(syn.seed_for(CONFIG_ID, 0, m, syn.KIND_WEIGHT), o, k)
        t, g = oracle.absmean_tensor(w)
        codes = oracle.pack_i2s(t)
        sc = np.full((o, k // 128), g, dtype=np.float32)
        x = syn.activations(syn.seed_for(CONFIG_ID, 0, m, syn.KIND_ACT), 1, k, outliers=True)
        cases.append((o, k, codes, sc, x))
    per_layer = sum(linear_bytes(o, k) for o, k, *_ in cases)

    def layer(pool=None):
        for o, k, codes, sc, x in cases:
            q, s, _ = oracle.quant_act(x)
            if pool is None:
                oracle.linear(codes, sc, k, q, s)
            else:
                step = (o + cores - 1) // cores
                list(pool.map(lambda r0: oracle.linear(codes[r0:r0 + step], sc[r0:r0 + step], k, q, s),
                              range(0, o, step)))

    def timed(pool=None):
        t0 = time.perf_counter()
        n = 0
        while True:
            layer(pool)
            n += 1
            dt = time.perf_counter() - t0
            if dt >= seconds:
                return n, dt

    n1, dt1 = timed()
    with cf.ThreadPoolExecutor(max_workers=cores) as pool:
        nN, dtN = timed(pool)
        # GEMM oracle: 64 tokens of 13824 x 2560, rows split over the cores.
        o, k, codes, sc, _ = cases[2]
        x = syn.activations(syn.seed_for(3, 0, 0, syn.KIND_ACT), 64, k)
        q, s, _ = oracle.quant_act(x)
        step = (o + cores - 1) // cores
        t0 = time.perf_counter()
        list(pool.map(lambda r0: oracle.linear(codes[r0:r0 + step], sc[r0:r0 + step], k, q, s), range(0, o, step)))
        dtg = time.perf_counter() - t0
    gemm_tops = 2.0 * 64 * o * k / dtg / 1e12
    return {"value": round(per_layer * n1 / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"layer 0 of the 30 (4 linears, all rows, batch 1), {n1} passes in {dt1:.1f} s on one core",
            "us_per_layer": round(dt1 / n1 * 1e6, 1),
            "all_cores": {"value": round(per_layer * nN / dtN / 1e9, 4), "unit": "GB/s", "cores": cores,
                          "us_per_layer": round(dtN / nN * 1e6, 1),
                          "sample": f"same layer, output rows split over {cores} threads, {nN} passes in {dtN:.1f} s"},
            "gemm_T2048_13824x2560_extrapolated": {
                "TOPS": round(gemm_tops, 6), "ms": round(dtg * 2048 / 64 * 1e3, 1), "cores": cores,
                "sample": "64 tokens timed on all cores, scaled linearly to T = 2048 (extrapolated)"},
            "cpu_model": cpu_model(), "nproc": cores}


# ------------------------------------------------------- small cases --

def run_case(args):
    """One kernel on one shape, for profiling: `--case gemv` runs
    bitnet_w2a8_gemv (batch `--batch`), `--case linear` bitnet_w2a8_linear,
    both over `--copies` distinct weights (so the weights exceed L2); `--case
    gemm` runs bitnet_w2a8_gemm on one weight (`--tokens`), `--case gemm_ws`
    bitnet_w2a8_gemm_ws (weights expanded into a workspace), `--case
    linear_ws` bitnet_w2a8_linear_ws (fp32 x in); `--case quant`
    bitnet_quant_act on `--tokens` rows; `--case seq` one bitnet_w2a8_linear_seq
    call over `--copies` linears of the shape; `--case step` the benchmark's
    step (timed from graph replays).  `--reps` passes, plain launches (no
    graph) except for `step`.  Prints one JSON line with the median time."""
    import torch

    import ternary_weight_absmax_b200 as b

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    o, k = args.rows, args.cols
    vec = args.case in ("gemv", "linear", "seq")
    if args.case == "step":
        args.copies = 1
    copies = args.copies if vec else 1
    ws = build_weights(b, torch, dev, copies, [("w", o, k)], 6)
    T = args.batch if vec else args.tokens
    x = torch.randn(T * k, dtype=torch.float32, device=dev)
    q = torch.empty(T * k, dtype=torch.int8, device=dev)
    s = torch.empty(T, dtype=torch.float32, device=dev)
    y = torch.empty(copies * T * o, dtype=torch.float32, device=dev)
    b.bitnet_quant_act(x, T, k, q, s)
    if args.case == "step":
        # The benchmark's step: 30 BitNet-2B-shaped layers, one sequence call.
        ws2 = build_weights(b, torch, dev, LAYERS, SHAPES, CONFIG_ID)
        xh, xd, xv = make_inputs(torch, dev, LAYERS, SHAPES, 1, CONFIG_ID)
        yd = torch.empty(sum(o_ for _, o_, _ in SHAPES) * LAYERS, dtype=torch.float32, device=dev)
        ys2, off = [], 0
        for l in range(LAYERS):
            for _, o_, _ in SHAPES:
                ys2.append(yd[off:off + o_])
                off += o_
        ents = linear_entries(ws2, LAYERS, SHAPES, xd, xv, ys2)
        calls = [lambda: b.bitnet_w2a8_linear_seq(ents)]
        copies = 1
    elif args.case == "seq":
        ents = [(ws[(c, "w")], x[:k], y[c * o:(c + 1) * o], -1) for c in range(copies)]
        calls = [lambda: b.bitnet_w2a8_linear_seq(ents)]
    elif args.case == "linear":
        calls = [lambda w=ws[(c, "w")]: b.bitnet_w2a8_linear(w, x, T, y[:T * o], q if T > 1 else None,
                                                              s if T > 1 else None) for c in range(copies)]
    elif args.case == "gemv":
        calls = [lambda w=ws[(c, "w")]: b.bitnet_w2a8_gemv(w, q, s, T, y[:T * o]) for c in range(copies)]
    elif args.case == "quant":
        calls = [lambda: b.bitnet_quant_act(x, T, k, q, s)]
    elif args.case == "gemm_ws":
        wsp = torch.empty(b.bitnet_w2a8_gemm_workspace_bytes(o, k), dtype=torch.uint8, device=dev)
        calls = [lambda: b.bitnet_w2a8_gemm_ws(ws[(0, "w")], q, s, T, y[:T * o], wsp)]
    elif args.case == "linear_ws":
        wsp = torch.empty(b.bitnet_w2a8_gemm_workspace_bytes(o, k), dtype=torch.uint8, device=dev)
        calls = [lambda: b.bitnet_w2a8_linear_ws(ws[(0, "w")], x, T, y[:T * o], q, s, wsp)]
    else:
        calls = [lambda: b.bitnet_w2a8_gemm(ws[(0, "w")], q, s, T, y[:T * o])]
    if args.case == "step":
        # Device time per step from graph replays: a plain call also times the
        # host-side marshalling of the 120 entries, which exceeds the kernel.
        Tm = Timer(torch, torch.cuda.Stream(device=dev), dev)
        med = Tm.ms(Tm.capture(calls[0]), 20, passes=max(1, args.reps)) * 1e3
    else:
        times = []
        for _ in range(args.reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for call in calls:
                call()
            e1.record()
            e1.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3 / copies)
        med = sorted(times)[len(times) // 2]
    assert b.bitnet_get_device_error() == b.BITNET_OK
    out = {"case": args.case, "out": o, "K": k, "T": T, "copies": copies, "us_per_linear": round(med, 3)}
    if args.case == "step":
        out = {"case": "step", "us_per_step": round(med, 3),
               "GB/s": round(fused_step_bytes() / (med * 1e-6) / 1e9, 1)}
    elif vec:
        nbytes = gemv_bytes(o, k, T) if args.case == "gemv" else linear_bytes(o, k, T)
        out["GB/s"] = round(nbytes / (med * 1e-6) / 1e9, 1)
    elif args.case == "quant":
        out["GB/s"] = round(5.0 * T * k / (med * 1e-6) / 1e9, 1)
    else:
        out["TOPS"] = round(2.0 * T * o * k / (med * 1e-6) / 1e12, 1)
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["gemv", "linear", "gemm", "gemm_ws", "linear_ws", "quant", "seq", "step"],
                    help="profile one kernel on one shape (step: the benchmark's sequence call)")
    ap.add_argument("--rows", type=int, default=13824)
    ap.add_argument("--cols", type=int, default=2560)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--tokens", type=int, default=2048)
    ap.add_argument("--copies", type=int, default=16)
    ap.add_argument("--reps", type=int, default=5)
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    import torch
    if args.warmup < 3:
        args.warmup = 3
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        out = run_ours(args, rank, world, dev)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline()
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
