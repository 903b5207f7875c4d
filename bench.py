"""Benchmark of the W2A8 (ternary i2_s x int8 absmax) linear layer on B200.

Default workload (one step): the decode linears of a BitNet-b1.58-2B-shaped
model at batch 1 -- 30 layers x {QKV 3840x2560, O 2560x2560, gate+up
13824x2560, down 2560x6912}, each with its own seeded weights and input.
Per linear: bitnet_w2a8_linear (fp32 x -> int8 q, s -> GEMV -> fp32 y, one
kernel).  The 120 C-ABI calls of a step are captured once in a CUDA graph and
the graph is replayed; the 520 MB of packed weights exceed the 126 MB L2, so
every step streams them from HBM.  The two-call path (bitnet_quant_act then
bitnet_w2a8_gemv) is timed the same way and reported beside it.

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

def build_weights(b, torch, dev, layers, shapes, seed_base):
    """Seeded fp32 N(0,1) weights drawn on the device, ternarised (per-tensor
    absmean) and packed by the library, then repacked.  Untimed setup."""
    ws = {}
    maxn = max(o * k for _, o, k in shapes)
    maxo, maxk = max(o for _, o, _ in shapes), max(k for _, _, k in shapes)
    wbuf = torch.empty(maxn, dtype=torch.float32, device=dev)
    cbuf = torch.empty(maxn // 4, dtype=torch.uint8, device=dev)
    sbuf = torch.empty(maxn // 128, dtype=torch.float32, device=dev)
    wsp = torch.empty(b.bitnet_ternarize_workspace_bytes(maxo, maxk) + 4096, dtype=torch.uint8, device=dev)
    gen = torch.Generator(device=dev)
    for l in range(layers):
        for m, (name, o, k) in enumerate(shapes):
            gen.manual_seed(seed_base ^ (l << 24) ^ (m << 16) ^ 1)
            w = wbuf[:o * k]
            w.normal_(generator=gen)
            b.bitnet_ternarize_absmean_device(w, o, k, b.BITNET_ABSMEAN_PER_TENSOR, cbuf[:o * k // 4],
                                              sbuf[:o * k // 128], wsp)
            data = torch.empty(b.bitnet_repacked_bytes(o, k), dtype=torch.uint8, device=dev)
            ws[(l, name)] = b.bitnet_repack_device(cbuf[:o * k // 4], sbuf[:o * k // 128], o, k, data)
    del wbuf, cbuf, sbuf, wsp
    return ws


def make_inputs(torch, dev, layers, shapes, B, seed_base, outliers=True):
    """x for every linear, one flat fp32 buffer (device) + pinned host copy."""
    total = sum(B * k for _, _, k in shapes) * layers
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed_base ^ 2)
    host = torch.randn(total, generator=gen, dtype=torch.float32)
    views, off = {}, 0
    for l in range(layers):
        for m, (name, o, k) in enumerate(shapes):
            x = host[off:off + B * k].view(B, k)
            if outliers:
                g2 = torch.Generator(device="cpu")
                g2.manual_seed(seed_base ^ (m << 16) ^ 3)
                ch = torch.randperm(k, generator=g2)[: k // 100]
                x[:, ch] *= 20.0
            views[(l, name)] = (off, B * k)
            off += B * k
    pinned = host.pin_memory()
    return pinned, pinned.to(dev), views


def run_ours(args, rank, world, dev):
    import numpy as np
    import torch

    import ternary_weight_absmax_b200 as b

    torch.cuda.set_device(dev)
    B = 1
    seed = 0xB17E7 ^ (CONFIG_ID << 40)
    weights = build_weights(b, torch, dev, LAYERS, SHAPES, seed)
    x_host, x_dev, xviews = make_inputs(torch, dev, LAYERS, SHAPES, B, seed)
    qbuf = {key: torch.empty(B * k, dtype=torch.int8, device=dev)
            for key in weights for (n, _, k) in SHAPES if n == key[1]}
    sbuf = {key: torch.empty(B, dtype=torch.float32, device=dev) for key in weights}
    ytot = sum(B * o for _, o, _ in SHAPES) * LAYERS
    y_dev = torch.empty(ytot, dtype=torch.float32, device=dev)
    y_host = torch.empty(ytot, dtype=torch.float32).pin_memory()
    yviews, off = {}, 0
    for l in range(LAYERS):
        for name, o, k in SHAPES:
            yviews[(l, name)] = y_dev[off:off + B * o]
            off += B * o

    stream = torch.cuda.Stream(device=dev)
    launches_per_step = 0

    def step(gemv_only=False, only=None):
        """Two C-ABI calls per linear: bitnet_quant_act, bitnet_w2a8_gemv."""
        n = 0
        for l in range(LAYERS):
            for name, o, k in SHAPES:
                if only is not None and name != only:
                    continue
                key = (l, name)
                xo, xn = xviews[key]
                if not gemv_only:
                    b.bitnet_quant_act(x_dev[xo:xo + xn], B, k, qbuf[key], sbuf[key])
                    n += 1
                b.bitnet_w2a8_gemv(weights[key], qbuf[key], sbuf[key], B, yviews[key])
                n += 1
        return n

    def fused_step():
        """One C-ABI call per linear: bitnet_w2a8_linear (quantise + GEMV)."""
        n = 0
        for l in range(LAYERS):
            for name, o, k in SHAPES:
                key = (l, name)
                xo, xn = xviews[key]
                b.bitnet_w2a8_linear(weights[key], x_dev[xo:xo + xn], B, yviews[key])
                n += 1
        return n

    # Warm the quantised inputs once so GEMV-only graphs read real q, s.
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize(dev)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            cnt = fn()
        return g, cnt

    g_step, launches_per_step = capture(fused_step)
    g_two, two_launches = capture(lambda: step())
    g_gemv, gemv_launches = capture(lambda: step(gemv_only=True))
    g_shape = {name: capture(lambda name=name: step(gemv_only=True, only=name))[0] for name, _, _ in SHAPES}
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed(graph, reps, pre=None):
        """Device ms per replay, CUDA events on the replay stream."""
        ms = []
        for _ in range(reps):
            if pre:
                with torch.cuda.stream(stream):
                    pre()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                graph.replay()
                e1.record(stream)
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        return ms

    clocks = ClockSampler(dev)
    clocks.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_step.replay()
    barrier()
    # ---- timed region: K steps back to back ----
    clocks.mark("t0")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            g_step.replay()
        e1.record(stream)
    e1.synchronize()
    barrier()
    clocks.mark("t1")
    step_ms_local = e0.elapsed_time(e1) / args.steps
    clocks.stop()

    # ---- the two-call path (bitnet_quant_act + bitnet_w2a8_gemv) ----
    two_ms = timed(g_two, max(3, min(50, args.steps)))
    two_ms_step = sorted(two_ms)[len(two_ms) // 2]
    # ---- GEMV-only replays (roofline of the dominant kernel) ----
    gemv_ms = timed(g_gemv, max(3, min(20, args.steps)))
    gemv_ms_per_step = sorted(gemv_ms)[len(gemv_ms) // 2]
    # ---- per-shape GEMV, L2 flushed before each pass ----
    per_shape = {}
    for name, o, k in SHAPES:
        ms = timed(g_shape[name], 7, pre=lambda: flush.fill_(1.0))
        med = sorted(ms)[len(ms) // 2] / LAYERS
        per_shape[name] = {"out": o, "K": k, "us": round(med * 1e3, 3),
                           "GB/s": round(gemv_bytes(o, k) / (med * 1e-3) / 1e9, 1)}
    del flush

    # ---- e2e: pinned host x -> device, the captured C-ABI calls, y -> host ----
    def e2e_once():
        with torch.cuda.stream(stream):
            x_dev.copy_(x_host, non_blocking=True)
            g_step.replay()
            y_host.copy_(y_dev, non_blocking=True)
    for _ in range(3):
        e2e_once()
    torch.cuda.synchronize(dev)
    e2e_steps = max(3, min(args.steps, 200))
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
    for _ in range(e2e_steps):
        e2e_once()
    with torch.cuda.stream(stream):
        f1.record(stream)
    f1.synchronize()
    e2e_ms_local = f0.elapsed_time(f1) / e2e_steps

    # ---- prefill GEMM (T=2048) ----
    prefill = run_prefill(b, torch, dev, stream, seed)
    small_batch = run_small_batch(b, torch, dev, stream, seed, weights)
    lut = run_lut(b, torch, dev, stream, weights)

    status = b.bitnet_get_device_error(stream.cuda_stream)
    if status != b.BITNET_OK:
        raise RuntimeError(f"device error after bench: {b.bitnet_status_string(status)}")

    gbytes, qbytes = step_bytes()
    per_rank_bytes = fused_step_bytes()
    step_ms, e2e_ms, gemv_ms_max, two_ms_max = reduce_max(
        [step_ms_local, e2e_ms_local, gemv_ms_per_step, two_ms_step], dev)
    value, _ = aggregate([step_ms] * world, [per_rank_bytes] * world)
    e2e_value, _ = aggregate([e2e_ms] * world, [per_rank_bytes] * world)

    peaks = read_peaks()
    # Dominant kernel: the batch-1 decode kernel behind bitnet_w2a8_linear, one
    # launch per linear of the step; its average launch time is the step time
    # (CUDA events on the launch stream, timed region above) over the launches.
    launch_us = step_ms * 1e3 / launches_per_step
    bytes_per_launch = per_rank_bytes / launches_per_step
    achieved = bytes_per_launch / (launch_us * 1e-6) / 1e9
    roofline = {"kernel": "decode_b1_kernel (bitnet_w2a8_linear, batch 1, uniform rows)", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
                "traffic": read_traffic(), "bytes_per_launch": round(bytes_per_launch, 1),
                "launch_us": round(launch_us, 3)}

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded N(0,1) weights ternarised on device; N(0,1) activations, 1% channels x20)",
        "path": "bitnet_w2a8_linear per linear (activation quantisation fused into the GEMV)",
        "config": {"workload": WORKLOAD, "shapes_out_x_K": [[o, k] for _, o, k in SHAPES], "layers": LAYERS,
                   "batch": B, "linears_per_step": LAYERS * len(SHAPES),
                   "l2": "inputs larger than L2 (520 MB packed weights per step); per-shape passes flush L2",
                   "graph": "the 120 C-ABI calls of a step captured in one CUDA graph",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "per_shape_gemv": per_shape,
        "two_call_step": {"ms_per_step": round(two_ms_max, 4),
                          "GB/s": round(aggregate([two_ms_max] * world, [gbytes + qbytes] * world)[0], 2),
                          "launches_per_step": two_launches,
                          "how": "bitnet_quant_act + bitnet_w2a8_gemv per linear, same graph replay timing"},
        "gemv_only_ms_per_step": round(gemv_ms_max, 4),
        "prefill": prefill,
        "small_batch_gemv": small_batch,
        "lut_gemv_b1": lut,
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": int(x_host.numel() * 4), "d2h_bytes_per_step": int(y_host.numel() * 4),
                "how": "pinned x copied in, graph of the step's C-ABI calls, y copied out, per step"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    return out


SMALL_BATCH = [("o", 2560, 2560), ("gate_up", 13824, 2560), ("wide", 20480, 3200)]
SMALL_BATCH_B = (1, 4, 16)


def run_small_batch(b, torch, dev, stream, seed, weights):
    """bitnet_w2a8_gemv at B = 1, 4, 16 on the standalone shapes: one call per
    distinct weight copy (30 copies of the step's O and gate+up weights, 12
    copies of 20480 x 3200), L2 flushed with a 512 MB write before each timed
    pass; median of 5 passes, us per call and algorithmic GB/s."""
    res = {}
    try:
        wide = build_weights(b, torch, dev, 12, [("wide", 20480, 3200)], seed ^ 0x99)
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
                with torch.cuda.stream(stream):
                    b.bitnet_quant_act(x, B, k, q, s)
                    for w in ws:
                        b.bitnet_w2a8_gemv(w, q, s, B, y)
                torch.cuda.synchronize(dev)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for w in ws:
                        b.bitnet_w2a8_gemv(w, q, s, B, y)
                ms = []
                for _ in range(5):
                    with torch.cuda.stream(stream):
                        flush.fill_(1.0)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    with torch.cuda.stream(stream):
                        e0.record(stream)
                        g.replay()
                        e1.record(stream)
                    e1.synchronize()
                    ms.append(e0.elapsed_time(e1) / len(ws))
                med = sorted(ms)[len(ms) // 2]
                res[name][f"B{B}"] = {"us": round(med * 1e3, 3),
                                      "GB/s": round(gemv_bytes(o, k, B) / (med * 1e-3) / 1e9, 1)}
                del g
        del flush, wide
    except Exception as e:  # reported beside the headline, never instead of it
        res["error"] = f"{type(e).__name__}: {e}"
    return res


def run_lut(b, torch, dev, stream, weights):
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
            calls = {"lut": lambda w: b.bitnet_w2a8_gemv_lut(w, q, s, y),
                     "dp4a": lambda w: b.bitnet_w2a8_gemv(w, q, s, 1, y)}
            res[name] = {"out": o, "K": k}
            for kind, call in calls.items():
                with torch.cuda.stream(stream):
                    b.bitnet_quant_act(x, 1, k, q, s)
                    for w in ws:
                        call(w)
                torch.cuda.synchronize(dev)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for w in ws:
                        call(w)
                ms = []
                for _ in range(5):
                    with torch.cuda.stream(stream):
                        flush.fill_(1.0)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    with torch.cuda.stream(stream):
                        e0.record(stream)
                        g.replay()
                        e1.record(stream)
                    e1.synchronize()
                    ms.append(e0.elapsed_time(e1) / len(ws))
                res[name][f"{kind}_us"] = round(sorted(ms)[2] * 1e3, 3)
                del g
        del flush
    except Exception as e:  # reported beside the headline, never instead of it
        res["error"] = f"{type(e).__name__}: {e}"
    return res


def run_prefill(b, torch, dev, stream, seed):
    res = {"T": PREFILL_T, "shapes": {}}
    try:
        weights = build_weights(b, torch, dev, 1, PREFILL, seed ^ 0x77)
        for name, o, k in PREFILL:
            w = weights[(0, name)]
            T = PREFILL_T
            x = torch.randn(T * k, dtype=torch.float32, device=dev)
            q = torch.empty(T * k, dtype=torch.int8, device=dev)
            s = torch.empty(T, dtype=torch.float32, device=dev)
            y = torch.empty(T * o, dtype=torch.float32, device=dev)
            with torch.cuda.stream(stream):
                b.bitnet_quant_act(x, T, k, q, s)
                for _ in range(3):
                    b.bitnet_w2a8_gemm(w, q, s, T, y)
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            reps = 10
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    b.bitnet_w2a8_gemm(w, q, s, T, y)
            ms = []
            for _ in range(5):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                e1.synchronize()
                ms.append(e0.elapsed_time(e1) / reps)
            med = sorted(ms)[len(ms) // 2]
            ops = 2.0 * T * o * k
            aq = []
            for _ in range(5):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    b.bitnet_quant_act(x, T, k, q, s)
                    e1.record(stream)
                e1.synchronize()
                aq.append(e0.elapsed_time(e1))
            res["shapes"][name] = {"out": o, "K": k, "gemm_us": round(med * 1e3, 2),
                                   "TOPS": round(ops / (med * 1e-3) / 1e12, 1),
                                   "act_quant_us": round(sorted(aq)[2] * 1e3, 2)}
            del g
        peaks = read_peaks()
        best = max(v["TOPS"] for v in res["shapes"].values())
        res["int8_peak_TOPS"] = peaks["int8_tops"]
        res["frac_of_int8_peak"] = round(best / peaks["int8_tops"], 4)
        res["peak_source"] = peaks["int8_source"]
    except Exception as e:  # the prefill figure is reported beside the headline, never instead of it
        res["error"] = f"{type(e).__name__}: {e}"
    return res


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        hbm, bf16 = float(d["hbm_gbs"]), float(d["bf16_tflops"])
        src = "measured (MEASURED_PEAKS.json: copy bandwidth)"
        isrc = "measured bf16 cuBLAS burst x 2 (nominal int8:bf16 dense ratio)"
    except (OSError, KeyError, ValueError):
        hbm, bf16 = 6650.0, 1590.0
        src = isrc = "fallback (6.65 TB/s, 1.59 PFLOP/s bf16)"
    return {"hbm_gbs": hbm, "int8_tops": 2.0 * bf16, "source": src, "int8_source": isrc}


def read_traffic():
    """DRAM bytes per decode-kernel launch (mean over the step's four shapes)
    from the committed ncu summary, if present."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(p) as f:
            return json.load(f).get("bytes_per_launch")
    except (OSError, ValueError):
        return None


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


def cpu_baseline(seconds=12.0):
    """The oracle timed on one host core on a bounded sample of the workload:
    layer 0's four linears, all output rows, batch 1, repeated for ~12 s."""
    import numpy as np

    import oracle
    import synthetic as syn

    oracle.build()
    B = 1
    cases = []
    for m, (name, o, k) in enumerate(SHAPES):
        w = syn.normal_matrix(syn.seed_for(CONFIG_ID, 0, m, syn.KIND_WEIGHT), o, k)
        t, g = oracle.absmean_tensor(w)
        codes = oracle.pack_i2s(t)
        sc = np.full((o, k // 128), g, dtype=np.float32)
        x = syn.activations(syn.seed_for(CONFIG_ID, 0, m, syn.KIND_ACT), B, k, outliers=True)
        cases.append((o, k, codes, sc, x))
    per_layer = sum(linear_bytes(o, k) for o, k, *_ in cases)
    t0 = time.perf_counter()
    n = 0
    while True:
        for o, k, codes, sc, x in cases:
            q, s, _ = oracle.quant_act(x)
            oracle.linear(codes, sc, k, q, s)
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    return {"value": round(per_layer * n / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"layer 0 of the 30 (4 linears, all rows, batch 1), {n} passes in {dt:.1f} s",
            "us_per_layer": round(dt / n * 1e6, 1)}


# ------------------------------------------------------- small cases --

def run_case(args):
    """One kernel on one shape, for profiling: `--case gemv` runs
    bitnet_w2a8_gemv and `--case linear` bitnet_w2a8_linear (activation
    quantisation fused) over `--copies` distinct weights (so the weights exceed
    L2), `--case gemm` runs bitnet_w2a8_gemm on one weight; `--reps` passes,
    plain launches (no graph).  Prints one JSON line with the median time."""
    import torch

    import ternary_weight_absmax_b200 as b

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    o, k = args.rows, args.cols
    seed = 0xB17E7 ^ 0x5A5A
    vec = args.case in ("gemv", "linear")
    copies = args.copies if vec else 1
    ws = build_weights(b, torch, dev, copies, [("w", o, k)], seed)
    T = args.batch if vec else args.tokens
    x = torch.randn(T * k, dtype=torch.float32, device=dev)
    q = torch.empty(T * k, dtype=torch.int8, device=dev)
    s = torch.empty(T, dtype=torch.float32, device=dev)
    y = torch.empty(T * o, dtype=torch.float32, device=dev)
    b.bitnet_quant_act(x, T, k, q, s)
    if args.case == "linear":
        def call(w, q_, s_, T_, y_):
            b.bitnet_w2a8_linear(w, x, T_, y_)
    else:
        call = b.bitnet_w2a8_gemv if args.case == "gemv" else b.bitnet_w2a8_gemm
    times = []
    for _ in range(args.reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for c in range(copies):
            call(ws[(c, "w")], q, s, T, y)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3 / copies)
    assert b.bitnet_get_device_error() == b.BITNET_OK
    med = sorted(times)[len(times) // 2]
    out = {"case": args.case, "out": o, "K": k, "T": T, "copies": copies, "us_per_launch": round(med, 3)}
    if vec:
        nbytes = gemv_bytes(o, k, T) if args.case == "gemv" else linear_bytes(o, k, T)
        out["GB/s"] = round(nbytes / (med * 1e-6) / 1e9, 1)
    else:
        out["TOPS"] = round(2.0 * T * o * k / (med * 1e-6) / 1e12, 1)
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["gemv", "linear", "gemm"], help="profile one kernel on one shape")
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
