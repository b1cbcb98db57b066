#!/usr/bin/env python
"""Benchmark of the SLQ weight-format hot path on B200 (one JSON line).

Headline workload: a Qwen3-8B-shaped decoder block at decode batch sizes --
hidden 4096, q/o 4096x4096 at 5 bits, k/v 1024x4096 at 8 bits, gate/up
12288x4096 and down 4096x12288 at 4 bits (asymmetric INT, group 128), X bf16
~ N(0,1) at M in {1, 4, 16}.  One step = the 7 dequantize-GEMMs of the block
at each of the three M, replayed as one CUDA graph; the projections that read
the same input in a decoder block run as one slq_gemm_group launch (q+k+v,
gate+up), so a step is 12 launches.  The metric
is packed-weight bytes streamed per second (codes + fp16 scales + uint8
zeros), whole job over all ranks.

The same line reports the other rows of the hot path, each timed with CUDA
events on its own stream: quantize+pack of the block's weights, the decode
sweep N=K=8192 at every b, the tiled GEMM at prefill sizes, and EAR/KL over
[4096 x 151936] logits.  Inputs are seeded synthetic stand-ins for the
pages' models (no checkpoints or datasets here).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl slq|reference]
  python bench.py --case SPEC [--steps K] [--warmup W]

--case runs one kernel of the path on its own (W untimed launches, then K
timed ones; with --graph the K calls replay as one CUDA graph) and prints
{"case", "avg_us", ...}: the command the profiles' ncu captures use.  SPEC is one of
  block                     the 12 decode launches of one Qwen3-8B block step
  gemv:N:K:b:M              one dequant-GEMM on the split-K GEMV kernel (M <= 16)
  decode:N:K:b:M            one dequant-GEMM on the stream-K decode kernel (M <= 16)
  tiled:N:K:b:M             one dequant-GEMM on the tiled tcgen05 kernel
  ear:T:V:tau               one EAR/KL reduction
  eartopk:T:V:tau:K         one top-K EAR/KL reduction
  quantize:N:K:b            one quantize+pack
  gridnoise:N:K:b           one grid-noise pass (gamma, asymmetric and symmetric SSE)
  gptq:N:K:T:b              one GPTQ encode of an [N, K] layer with T calibration rows

--impl reference times the CPU oracle (the plain reference implementation
of the same arithmetic) on a bounded sample of the same workload, on the
host cores, and reports the same metric.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GROUP = 128
L2_BYTES = 126 * 2**20

# Qwen3-8B-shaped block: (name, N, K, bits)
QWEN3_8B_BLOCK = [("q", 4096, 4096, 5), ("k", 1024, 4096, 8), ("v", 1024, 4096, 8),
                  ("o", 4096, 4096, 5), ("gate", 12288, 4096, 4), ("up", 12288, 4096, 4),
                  ("down", 4096, 12288, 4)]
DECODE_MS = (1, 4, 16)
# Launches of one block at one M: the projections that read the same input
# in a decoder block run as one grouped launch (q, k, v; gate, up).
BLOCK_LAUNCHES = ((0, 1, 2), (3,), (4, 5), (6,))
METRIC = "W{2-8}A16 GEMM weight GB/s (% HBM peak) & TFLOP/s per b and M; EAR/KL GB/s"
WORKLOAD = ("Qwen3-8B-shaped decoder block decode: q/o 4096x4096 b5, k/v 1024x4096 b8, "
            "gate/up 12288x4096 b4, down 4096x12288 b4, asymmetric INT g128; "
            "M in {1,4,16}; per M: q+k+v in one slq_gemm_group launch, o, gate+up in one, down "
            "(12 launches per step, one CUDA graph); independent X per projection")


def weight_bytes(N, K, bits):
    return N * K * bits // 8 + N * (K // GROUP) * 3


BLOCK_BYTES = sum(weight_bytes(N, K, b) for _, N, K, b in QWEN3_8B_BLOCK)

# GPTQ rows: the oracle's timed sample, and a 4096 x 4096 projection with the
# pages' 512 calibration rows per layer order of magnitude.
GPTQ_SHAPES = [(256, 1024, 256, 4), (4096, 4096, 512, 4)]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------
# Clock sampling (nvidia-smi) during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while a region runs.

    NVML is polled every millisecond from a thread (the timed regions here last
    tens of milliseconds); nvidia-smi's 100 ms loop is the fallback when NVML
    cannot be loaded.  Only reads settings, never changes them."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clocks-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, gpu_index: int, pci_bus_id: str | None = None):
        self.gpu = gpu_index
        self.pci = pci_bus_id
        self.proc = None
        self.lines = []
        self.thread = None
        self.stop_flag = threading.Event()
        self.samples = []  # (sm_mhz, max_mhz, reasons bitmask)
        self.nvml = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByPciBusId(self.pci) if self.pci
                 else pynvml.nvmlDeviceGetHandleByIndex(self.gpu))
            self.nvml = (pynvml, h)
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _poll(self):
        pynvml, h = self.nvml
        smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop_flag.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, smax, rs))
            except Exception:
                pass
            time.sleep(0.001)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        self.stop_flag.set()
        if self.nvml is not None:
            if self.thread:
                self.thread.join(timeout=2)
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": "nvml"}
            reasons = sorted({nm for _, _, rs in self.samples for bit, nm in self.REASONS.items() if rs & bit})
            return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                    "sm_max_mhz": max(s[1] for s in self.samples), "reasons": reasons,
                    "samples": len(self.samples), "source": "nvml, 1 ms polling during the timed region"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
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
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi -lms 100"}


# ----------------------------------------------------------------------------
# CUDA events as graph nodes (cudaEventRecordExternal) for per-launch timing
# ----------------------------------------------------------------------------
class GraphEvents:
    """Event-record nodes inside a captured graph, read after replay."""

    def __init__(self, n: int):
        import nvidia.cuda_runtime as cr
        path = os.path.join(list(cr.__path__)[0], "lib", "libcudart.so.12")
        self.rt = ctypes.CDLL(path)
        self.events = []
        for _ in range(n):
            ev = ctypes.c_void_p()
            if self.rt.cudaEventCreate(ctypes.byref(ev)) != 0:
                raise RuntimeError("cudaEventCreate failed")
            self.events.append(ev)

    def record(self, i: int, stream_handle: int):
        rc = self.rt.cudaEventRecordWithFlags(self.events[i], ctypes.c_void_p(stream_handle), 1)
        if rc != 0:
            raise RuntimeError(f"cudaEventRecordWithFlags failed ({rc})")

    def elapsed_ms(self, i: int, j: int) -> float:
        ms = ctypes.c_float()
        rc = self.rt.cudaEventElapsedTime(ctypes.byref(ms), self.events[i], self.events[j])
        if rc != 0:
            raise RuntimeError(f"cudaEventElapsedTime failed ({rc})")
        return ms.value


# ----------------------------------------------------------------------------
# The SLQ arm
# ----------------------------------------------------------------------------
def run_slq(args, rank, world, local_rank):
    import torch
    import synth
    import weight_only_mixed_b200 as slq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, tc_peak_sus, peak_kind = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    sh = stream.cuda_stream

    # ---- setup (untimed): quantize the block's weights, rotated copies -------
    R = max(2, int(np.ceil(4 * L2_BYTES / BLOCK_BYTES)))
    layers = []  # layers[r][i] = QuantizedWeight
    for r in range(R):
        copy = []
        for i, (name, N, K, b) in enumerate(QWEN3_8B_BLOCK):
            W = synth.weights_torch(N, K, seed=synth.SEED_WEIGHTS + 10 * i + 1000 * r + rank, device=dev)
            copy.append(slq.quantize(W, b))
            del W
        layers.append(copy)
    X = {M: [synth.activations_torch(M, K, seed=synth.SEED_X + 10 * i + M, device=dev)
             for i, (_, N, K, b) in enumerate(QWEN3_8B_BLOCK)] for M in DECODE_MS}
    Y = {M: [torch.empty((M, N), dtype=torch.bfloat16, device=dev)
             for (_, N, K, b) in QWEN3_8B_BLOCK] for M in DECODE_MS}
    torch.cuda.synchronize()

    n_launch = len(DECODE_MS) * len(BLOCK_LAUNCHES)

    def block_launch(M, r, grp, xs=None):
        xs = xs if xs is not None else X[M]
        if len(grp) == 1:
            i = grp[0]
            slq.gemm(xs[i], layers[r][i], out=Y[M][i], stream=stream)
        else:
            slq.gemm_group([(xs[i], layers[r][i]) for i in grp], outs=[Y[M][i] for i in grp],
                           stream=stream)
    try:
        gev = [GraphEvents(n_launch + 1) for _ in range(R)]
    except Exception:
        gev = None

    def step_body(r, ev=None):
        k = 0
        for M in DECODE_MS:
            for grp in BLOCK_LAUNCHES:
                if ev is not None:
                    ev.record(k, sh)
                block_launch(M, r, grp)
                k += 1
        if ev is not None:
            ev.record(k, sh)

    # Warm up eagerly once (device attributes, first launches), then capture.
    # The timed graphs hold only the kernels, so consecutive launches overlap
    # (programmatic dependent launch); a second set with an event between
    # kernels gives the per-launch durations and is replayed after the timed
    # region.
    step_body(0)
    torch.cuda.synchronize()
    graphs, ev_graphs = [], []
    for r in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step_body(r)
        graphs.append(g)
        if gev is not None:
            ge = torch.cuda.CUDAGraph()
            try:
                with torch.cuda.graph(ge, stream=stream):
                    step_body(r, gev[r])
                ev_graphs.append(ge)
            except Exception:
                gev = None
    torch.cuda.synchronize()
    for g in graphs:  # first replay uploads the graph
        g.replay()
    torch.cuda.synchronize()

    dist = None
    if world > 1:
        import torch.distributed as dist

    for s in range(args.warmup):
        graphs[s % R].replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(dev)
    pci = None
    if all(hasattr(props, a) for a in ("pci_domain_id", "pci_bus_id", "pci_device_id")):
        pci = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    try:
        smi_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[local_rank])
    except (ValueError, IndexError):
        smi_index = local_rank
    clocks = ClockSampler(smi_index, pci)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    reps = max(1, args.repeat)
    t0.record(stream)
    for s in range(args.steps * reps):
        graphs[s % R].replay()
    t1.record(stream)
    t1.synchronize()
    ms_total = t0.elapsed_time(t1)
    clk = clocks.stop()
    ms_step = ms_total / (args.steps * reps)
    ms_step = max_over_ranks(ms_step, dist, dev)
    if dist:
        dist.barrier()

    value = world * 3 * BLOCK_BYTES / (ms_step * 1e-3) / 1e9  # GB/s, whole job

    # Per-launch durations of the decode kernel: one replay of each
    # event-instrumented graph after the timed region.
    per_m = {}
    kernel_ms = None
    if gev is not None and len(ev_graphs) == R:
        for ge in ev_graphs:
            ge.replay()
        torch.cuda.synchronize()
        tot_bytes, tot_ms = 0.0, 0.0
        for r in range(R):
            k = 0
            for M in DECODE_MS:
                for grp in BLOCK_LAUNCHES:
                    d = gev[r].elapsed_ms(k, k + 1)
                    wb = sum(weight_bytes(*QWEN3_8B_BLOCK[i][1:]) for i in grp)
                    per_m.setdefault(M, [0.0, 0.0])
                    per_m[M][0] += wb
                    per_m[M][1] += d
                    tot_bytes += wb
                    tot_ms += d
                    k += 1
        kernel_ms = tot_ms / (R * n_launch)
    # In the timed graph the 12 launches of a step follow each other
    # (programmatic dependent launch lets each start while the previous one
    # drains), so the duration of a launch there is the step time / 12 and the
    # kernel's achieved rate is the step's rate.  The serialised replay above
    # (event nodes between launches) gives each launch alone, for reference.
    achieved = 3 * BLOCK_BYTES / (ms_step * 1e-3) / 1e9
    inflight_launch_us = ms_step * 1e3 / n_launch
    breakdown = {f"M={M}": {"isolated_weight_GBps": round(v[0] / (v[1] * 1e-3) / 1e9, 1),
                            "isolated_frac_hbm": round(v[0] / (v[1] * 1e-3) / 1e9 / hbm_peak, 3)}
                 for M, v in per_m.items()}

    # ---- e2e: public Python API, host buffers, copies inside the timed region.
    # Each step's 21 activation inputs sit in one pinned host buffer and are
    # copied to one device buffer with a single copy; the 21 outputs are views
    # of one device buffer read back with a single copy.
    x_len = {(M, i): M * QWEN3_8B_BLOCK[i][2] for M in DECODE_MS for i in range(len(QWEN3_8B_BLOCK))}
    y_len = {(M, i): M * QWEN3_8B_BLOCK[i][1] for M in DECODE_MS for i in range(len(QWEN3_8B_BLOCK))}
    Xh = torch.empty(sum(x_len.values()), dtype=torch.bfloat16).pin_memory()
    Yh = torch.empty(sum(y_len.values()), dtype=torch.bfloat16).pin_memory()
    Xd = torch.empty_like(Xh, device=dev)
    Yd = torch.empty_like(Yh, device=dev)
    Xv, Yv, o = {M: [] for M in DECODE_MS}, {M: [] for M in DECODE_MS}, 0
    for M in DECODE_MS:
        for i, (_, N, K, b) in enumerate(QWEN3_8B_BLOCK):
            Xh[o:o + M * K].copy_(X[M][i].reshape(-1).cpu())
            Xv[M].append(Xd[o:o + M * K].view(M, K))
            o += M * K
    o = 0
    for M in DECODE_MS:
        for i, (_, N, K, b) in enumerate(QWEN3_8B_BLOCK):
            Yv[M].append(Yd[o:o + M * N].view(M, N))
            o += M * N
    h2d = Xh.numel() * 2
    d2h = Yh.numel() * 2

    def e2e_step(r):
        Xd.copy_(Xh, non_blocking=True)
        for M in DECODE_MS:
            for grp in BLOCK_LAUNCHES:
                if len(grp) == 1:
                    slq.gemm(Xv[M][grp[0]], layers[r][grp[0]], out=Yv[M][grp[0]], stream=stream)
                else:
                    slq.gemm_group([(Xv[M][i], layers[r][i]) for i in grp], outs=[Yv[M][i] for i in grp],
                                   stream=stream)
        Yh.copy_(Yd, non_blocking=True)
        stream.synchronize()

    for s_ in range(max(1, args.warmup)):
        e2e_step(s_ % R)
    e2e_steps = max(3, args.steps)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s_ in range(e2e_steps):
        e2e_step(s_ % R)
    e1.record(stream)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    e2e_value = world * 3 * BLOCK_BYTES / (e2e_ms * 1e-3) / 1e9

    rows = {}
    if not args.headline_only:
        rows = other_rows(args, slq, synth, torch, dev, stream, hbm_peak, tc_peak, rank)

    # free the rotated copies before the CPU baseline
    del layers, graphs, ev_graphs
    torch.cuda.synchronize()

    out = None
    if rank == 0:
        cpu = cpu_baseline(args) if (world == 1 and not args.no_cpu) else None
        out = {
            "metric": METRIC,
            "value": round(value, 1),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded skewed-Gaussian weights, N(0,1) activations; no checkpoints)",
            "config": {
                "workload": WORKLOAD,
                "block_weight_bytes": BLOCK_BYTES,
                "bytes_per_step": 3 * BLOCK_BYTES,
                "l2": f"inputs larger than L2: {R} rotated weight copies ({R * BLOCK_BYTES / 2**20:.0f} MiB > 126 MiB L2)",
                "parallelism": f"replicas x{world} (independent layers per rank, no collective)",
                "repeat": reps,
            },
            "roofline": {
                "bound": "hbm",
                "kernel": "gemm_gemv_group_kernel / gemm_gemv_kernel<b> (split-K GEMV: packed W streamed by cp.async through per-warp shared-memory rings; the codes masked in place are exact subnormal bf16 mma.sync A fragments, the activations scaled by 2^(E-c) per group, the zero point folded out through a constant-A mma, fp32 group-scaled accumulate, deterministic in-CTA split-K; M<=16)",
                "achieved": round(achieved, 1),
                "peak": hbm_peak,
                "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4),
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6650 GB/s",
                "algorithmic_bytes": "N*K*(b/8 + 3/128) per launch (codes + fp16 scale + u8 zero); "
                                     f"{3 * BLOCK_BYTES // n_launch} bytes per launch on average",
                "avg_launch_us": round(inflight_launch_us, 3),
                "avg_launch_us_how": "timed graph: ms_per_step / 12 launches (the launches of a step run back to back)",
                "isolated_launch_us": round(kernel_ms * 1e3, 3) if kernel_ms else None,
                "isolated_GBps": round(3 * BLOCK_BYTES / (kernel_ms * n_launch * 1e-3) / 1e9, 1) if kernel_ms else None,
                "traffic": decode_traffic(),
                "per_M": breakdown,
            },
            "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "how": "public Python API (slq.gemm_group for q+k+v and gate+up, slq.gemm for o and down); per step one pinned-host-to-device copy of all 21 inputs, the 12 calls on views of that buffer, one device-to-pinned-host copy of all 21 outputs"},
            "gpu_launches": n_launch * args.steps * reps,
            "clocks": clk,
            "rows": rows,
        }
        if cpu is not None:
            out["cpu_baseline"] = cpu
    return out


def max_over_ranks(value: float, dist, device) -> float:
    """The largest `value` over all ranks (a replicated job takes as long as
    its slowest rank); `value` itself when there is no process group."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_ms(torch, stream, fn, iters, warm=2):
    for _ in range(warm):
        fn()
    stream.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / iters


def other_rows(args, slq, synth, torch, dev, stream, hbm_peak, tc_peak, rank):
    rows = {}
    # Quantize + pack of the block's 7 weights (reads bf16, writes packed).
    Ws = [synth.weights_torch(N, K, seed=90 + i, device=dev) for i, (_, N, K, b) in enumerate(QWEN3_8B_BLOCK)]
    outs = [slq.empty_quantized(N, K, b, dev) for (_, N, K, b) in QWEN3_8B_BLOCK]

    def qstep():
        for W, q, (_, N, K, b) in zip(Ws, outs, QWEN3_8B_BLOCK):
            slq.quantize(W, b, out=q, stream=stream)

    ms = time_ms(torch, stream, qstep, 10)
    qbytes = sum(N * K * 2 + weight_bytes(N, K, b) for _, N, K, b in QWEN3_8B_BLOCK)
    rows["quantize_block"] = {"GBps": round(qbytes / (ms * 1e-3) / 1e9, 1),
                              "frac_hbm": round(qbytes / (ms * 1e-3) / 1e9 / hbm_peak, 3),
                              "us": round(ms * 1e3, 2), "bytes": qbytes}
    # Grid noise (gamma, asymmetric and symmetric SSE) of the same 7 weights.
    gouts = [[torch.empty((N, K // 128), dtype=torch.float32, device=dev) for _ in range(3)]
             for (_, N, K, b) in QWEN3_8B_BLOCK]
    L = slq.lib()

    def gstep():
        for W, o, (_, N, K, b) in zip(Ws, gouts, QWEN3_8B_BLOCK):
            rc = L.slq_grid_noise(W.data_ptr(), N, K, b, o[0].data_ptr(), o[1].data_ptr(),
                                  o[2].data_ptr(), None, stream.cuda_stream)
            assert rc == 0

    ms = time_ms(torch, stream, gstep, 10)
    gbytes = sum(N * K * 2 + 12 * N * (K // 128) for _, N, K, b in QWEN3_8B_BLOCK)
    rows["grid_noise_block"] = {"GBps": round(gbytes / (ms * 1e-3) / 1e9, 1),
                                "frac_hbm": round(gbytes / (ms * 1e-3) / 1e9 / hbm_peak, 3),
                                "us": round(ms * 1e3, 2), "bytes": gbytes}
    del Ws, outs, gouts

    # Decode sweep N = K = 8192 at every b, M in {1, 16}.
    sweep = {}
    N = K = 8192
    for b in range(2, 9):
        nrot = max(2, int(np.ceil(4 * L2_BYTES / weight_bytes(N, K, b))))
        qws = [slq.quantize(synth.weights_torch(N, K, seed=700 + b + 10 * r, device=dev), b) for r in range(nrot)]
        for M in (1, 16):
            Xs = synth.activations_torch(M, K, seed=800 + M, device=dev)
            Ys = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            it = [0]

            def f():
                slq.gemm(Xs, qws[it[0] % nrot], out=Ys, stream=stream)
                it[0] += 1

            slq.gemm(Xs, qws[0], out=Ys, stream=stream)  # sizes the workspace before capture
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for r in range(nrot):
                    slq.gemm(Xs, qws[r], out=Ys, stream=stream)
            ms = time_ms(torch, stream, g.replay, 20) / nrot
            gbps = weight_bytes(N, K, b) / (ms * 1e-3) / 1e9
            sweep[f"b{b}_M{M}"] = {"GBps": round(gbps, 1), "frac_hbm": round(gbps / hbm_peak, 3),
                                   "TFLOPs": round(2 * M * N * K / (ms * 1e-3) / 1e12, 2),
                                   "us": round(ms * 1e3, 2)}
        del qws
    rows["decode_sweep_8192"] = sweep

    # Config 0: one 1024 x 1024 layer at b = 4, M = 8.  Its 0.55 MB of packed
    # weights stay in L2 across launches, so the rate is an L2 figure, flagged.
    N = K = 1024
    q0 = slq.quantize(synth.weights_torch(N, K, seed=synth.SEED_WEIGHTS, device=dev), 4)
    X0 = synth.activations_torch(8, K, seed=synth.SEED_X, device=dev)
    Y0 = torch.empty((8, N), dtype=torch.bfloat16, device=dev)
    slq.gemm(X0, q0, out=Y0, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(20):
            slq.gemm(X0, q0, out=Y0, stream=stream)
    ms = time_ms(torch, stream, g.replay, 20) / 20
    gbps = weight_bytes(N, K, 4) / (ms * 1e-3) / 1e9
    rows["config0_1024x1024_b4_M8"] = {"GBps": round(gbps, 1), "frac_hbm": round(gbps / hbm_peak, 3),
                                       "us": round(ms * 1e3, 2), "l2_resident": True,
                                       "note": "0.55 MB of weights re-read from L2 by 20 back-to-back launches"}
    del g, q0, X0, Y0

    # Tiled (prefill) GEMM: N = K = 8192 at M in {1024, 4096}, and the
    # Llama-3.3-70B-shaped block at M = 2048; TFLOP/s on 2*M*N*K.
    pre = {}
    N = K = 8192
    for b in range(2, 9):
        qw = slq.quantize(synth.weights_torch(N, K, seed=900 + b, device=dev), b)
        for M in (1024, 4096):
            Xp = synth.activations_torch(M, K, seed=901, device=dev)
            Yp = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ms = time_ms(torch, stream, lambda: slq.gemm(Xp, qw, out=Yp, stream=stream), 10)
            tf = 2 * M * N * K / (ms * 1e-3) / 1e12
            pre[f"sweep8192_b{b}_M{M}"] = {"TFLOPs": round(tf, 1), "frac_tensor": round(tf / tc_peak, 3),
                                           "us": round(ms * 1e3, 1)}
            del Xp, Yp
        del qw
    # The sizes reported only, M = 64 and 256 on 8192^2 (memory-bound for
    # b >= 3): weights rotated over more than L2, launches replayed from a graph.
    N = K = 8192
    for b in range(2, 9):
        nrot = max(2, int(np.ceil(4 * L2_BYTES / weight_bytes(N, K, b))))
        qws = [slq.quantize(synth.weights_torch(N, K, seed=920 + b + 10 * r, device=dev), b) for r in range(nrot)]
        for M in (64, 256):
            Xp = synth.activations_torch(M, K, seed=921, device=dev)
            Yp = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            slq.gemm(Xp, qws[0], out=Yp, stream=stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for r in range(nrot):
                    slq.gemm(Xp, qws[r], out=Yp, stream=stream)
            ms = time_ms(torch, stream, g.replay, 10) / nrot
            gbps = weight_bytes(N, K, b) / (ms * 1e-3) / 1e9
            tf = 2 * M * N * K / (ms * 1e-3) / 1e12
            pre[f"sweep8192_b{b}_M{M}"] = {"GBps": round(gbps, 1), "frac_hbm": round(gbps / hbm_peak, 3),
                                           "TFLOPs": round(tf, 1), "frac_tensor": round(tf / tc_peak, 3),
                                           "us": round(ms * 1e3, 1)}
            del g, Xp, Yp
        del qws
    # The Llama-3.3-70B-shaped block (683 MB of packed weights, more than
    # L2) at M = 1, 16, 64 and 2048: seven launches per step.
    llama = [(8192, 8192, 7), (1024, 8192, 8), (1024, 8192, 8), (8192, 8192, 7), (28672, 8192, 6),
             (28672, 8192, 6), (8192, 28672, 6)]
    qws = [slq.quantize(synth.weights_torch(N, K, seed=950 + i, device=dev), b) for i, (N, K, b) in enumerate(llama)]
    wbytes = sum(weight_bytes(N, K, b) for (N, K, b) in llama)
    for M in (1, 16, 64, 2048):
        Xs = [synth.activations_torch(M, K, seed=960 + i, device=dev) for i, (N, K, b) in enumerate(llama)]
        Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for (N, K, b) in llama]

        def block():
            for x, q, y in zip(Xs, qws, Ys):
                slq.gemm(x, q, out=y, stream=stream)

        block()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            block()
        ms = time_ms(torch, stream, g.replay, 5)
        flops = sum(2 * M * N * K for (N, K, b) in llama)
        tf = flops / (ms * 1e-3) / 1e12
        gbps = wbytes / (ms * 1e-3) / 1e9
        pre[f"llama70b_block_M{M}"] = {"GBps": round(gbps, 1), "frac_hbm": round(gbps / hbm_peak, 3),
                                       "TFLOPs": round(tf, 1), "frac_tensor": round(tf / tc_peak, 3),
                                       "us": round(ms * 1e3, 1)}
        del g, Xs, Ys
    del qws
    rows["tiled_prefill"] = pre

    # EAR / KL over [4096 x 151936] bf16 logits, tau 1.0 and 0.7.
    T, V = 4096, 151936
    a, bq = synth.logits_torch(T, V, device=dev)
    ear = torch.empty(T, dtype=torch.float32, device=dev)
    kl = torch.empty(T, dtype=torch.float32, device=dev)
    em = torch.empty((), dtype=torch.float64, device=dev)
    km = torch.empty((), dtype=torch.float64, device=dev)
    L = slq.lib()
    for tau in (1.0, 0.7):
        def f():
            rc = L.slq_ear_kl(a.data_ptr(), bq.data_ptr(), T, V, tau, ear.data_ptr(), kl.data_ptr(),
                              em.data_ptr(), km.data_ptr(), None, stream.cuda_stream)
            assert rc == 0
        ms = time_ms(torch, stream, f, 5, warm=1)
        nbytes = 2 * T * V * 2
        rows[f"ear_kl_tau{tau}"] = {"GBps": round(nbytes / (ms * 1e-3) / 1e9, 1),
                                    "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm_peak, 3),
                                    "us": round(ms * 1e3, 1), "ear_mean": round(em.item(), 6),
                                    "kl_mean": round(km.item(), 7)}
    # Top-K form (K = 10, the pages' evaluation), one pass over the logits.
    for tau in (1.0,):
        def f():
            rc = L.slq_ear_kl_topk(a.data_ptr(), bq.data_ptr(), T, V, 10, tau, ear.data_ptr(),
                                   kl.data_ptr(), em.data_ptr(), km.data_ptr(), None, stream.cuda_stream)
            assert rc == 0
        ms = time_ms(torch, stream, f, 5, warm=1)
        nbytes = 2 * T * V * 2
        rows[f"ear_kl_top10_tau{tau}"] = {"GBps": round(nbytes / (ms * 1e-3) / 1e9, 1),
                                          "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm_peak, 3),
                                          "us": round(ms * 1e3, 1), "ear_mean": round(em.item(), 6),
                                          "kl_mean": round(km.item(), 7)}
    del a, bq

    # GPTQ encode of one layer (slq_gptq: H, factorizations, column encode),
    # on the oracle's sample shape and on a 4096 x 4096 projection.
    for (N, K, T, b) in GPTQ_SHAPES:
        W = synth.weights_torch(N, K, seed=800 + N, device=dev)
        X = torch.from_numpy(synth.calibration(T, K, seed=801 + K).view(np.int16)).to(dev).view(torch.bfloat16)
        out = slq.empty_quantized(N, K, b, dev)
        ws = torch.empty(slq.gptq_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        slq.gptq(W, X, b, out=out, workspace=ws, stream=stream)
        ms = time_ms(torch, stream, lambda: slq.gptq(W, X, b, out=out, workspace=ws, stream=stream), 3, warm=1)
        rows[f"gptq_{N}x{K}_T{T}_b{b}"] = {"ms": round(ms, 2), "launches": 6 * (K // 32) + 2 * (K // 128) + 3}
        del W, X, out, ws
    return rows


# ----------------------------------------------------------------------------
# CPU baseline / reference arm: the oracle on a bounded sample, on one core
# and on every core this process may use (a spawn pool, one worker per core,
# each timing the oracle on its own slice of the sample)
# ----------------------------------------------------------------------------
def _host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _gemm_work(i, row0, rows):
    """Rows [row0, row0 + rows) of projection i of the Qwen3-8B block, quantized
    by the oracle (untimed), with that projection's activations at each M."""
    import oracle
    import synth
    name, N, K, b = QWEN3_8B_BLOCK[i]
    w = synth.weights(N if rows is None else min(rows, N - row0), K, seed=synth.SEED_WEIGHTS + 10 * i + row0)
    packed, scales, zeros, _ = oracle.quantize(w, b)
    xs = {M: synth.activations(M, K, seed=synth.SEED_X + M + i) for M in DECODE_MS}
    return packed.shape[0], K, b, packed, scales, zeros, xs


def _gemm_job(rows):
    """The per-worker GEMM sample: the first `rows` output rows of each of the
    7 projections, at every decode M."""
    return ("gemm", [(i, 0, min(N, rows)) for i, (_, N, K, b) in enumerate(QWEN3_8B_BLOCK)], 1)


def _quantize_job(rows):
    return ("quantize", [(i, 0, rows) for i in range(len(QWEN3_8B_BLOCK))])


def _ear_job(tokens, k=0):
    return ("ear", tokens, 151936, 3000 + 2 * k)


def _worker(job, barrier, queue):
    """Build the job's inputs, wait for every worker, then run and time it."""
    _oracle_job_prepared(job, barrier, queue)


def _oracle_job_prepared(job, barrier, queue):
    import oracle
    import synth
    kind = job[0]
    if kind == "gemm":
        work = [_gemm_work(i, r0, n) for i, r0, n in job[1]]

        def run():
            nb = 0
            for n, K, b, packed, scales, zeros, xs in work:
                for M in DECODE_MS:
                    oracle.gemm(xs[M], packed, scales, zeros, K, b)
                    nb += weight_bytes(n, K, b)
            return nb
    elif kind == "quantize":
        ws = [(synth.weights(n, QWEN3_8B_BLOCK[i][2], seed=97 + i + r0), QWEN3_8B_BLOCK[i][3]) for i, r0, n in job[1]]

        def run():
            nb = 0
            for w, b in ws:
                oracle.quantize(w, b)
                nb += w.size * 2 + weight_bytes(w.shape[0], w.shape[1], b)
            return nb
    elif kind == "gptq":
        _, N, K, T, b = job
        w = synth.weights(N, K, seed=800 + N)
        x = synth.calibration(T, K, seed=801 + K)

        def run():
            oracle.gptq(w, x, b)
            return 1  # layers
    else:
        _, tokens, V, seed = job
        a, bq = synth.logits(tokens, V, seed=seed, noise_seed=seed + 1)

        def run():
            oracle.ear_kl(a, bq, 1.0)
            return 2 * tokens * V * 2
    if barrier is not None:
        barrier.wait(timeout=600)
    t0 = time.time()
    nb = run()
    t1 = time.time()
    if queue is not None:
        queue.put((nb, t0, t1))
    return nb, t0, t1


def _run_parallel(jobs):
    """Run each job in its own spawned process (one per core), all starting at
    a barrier once their inputs are built; returns (bytes, span seconds)."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")  # never fork a process that may hold a CUDA context
    barrier = ctx.Barrier(len(jobs))
    queue = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(job, barrier, queue)) for job in jobs]
    for p in procs:
        p.start()
    res = [queue.get(timeout=900) for _ in procs]
    for p in procs:
        p.join()
    return sum(r[0] for r in res), max(r[2] for r in res) - min(r[1] for r in res)


def oracle_rates(rows_per_layer: int, all_cores: bool):
    """Oracle throughput for the decode GEMM, quantize+pack and EAR/KL: one
    job on one core, and one job per core on every core this process may use."""
    cores = _host_cores()
    out = {"cores_available": cores}
    t_start = time.perf_counter()
    jobs = {"gemm": _gemm_job(rows_per_layer), "quantize": _quantize_job(64), "ear": _ear_job(8)}
    for name, job in jobs.items():
        nb, t0, t1 = _oracle_job_prepared(job, None, None)
        out[f"{name}_1core"] = nb / (t1 - t0) / 1e9
    # GPTQ: seconds per layer on one core (its factorizations are not split
    # over rows, so there is no all-core form of the same job).
    _, t0, t1 = _oracle_job_prepared(("gptq",) + GPTQ_SHAPES[0], None, None)
    out["gptq_1core_s"] = t1 - t0
    if all_cores and cores > 1:
        for name, job in jobs.items():
            par = [job if name != "ear" else _ear_job(8, k) for k in range(cores)]
            nb, span = _run_parallel(par)
            out[f"{name}_allcore"] = nb / span / 1e9
    out["wall_s"] = time.perf_counter() - t_start
    return out


def cpu_baseline(args):
    rates = oracle_rates(args.cpu_rows, not args.cpu_single)
    cores = rates["cores_available"]
    allc = "gemm_allcore" in rates
    r = lambda v: None if v is None else round(v, 5)
    return {
        "value": r(rates["gemm_allcore"] if allc else rates["gemm_1core"]), "unit": "GB/s",
        "cores": cores if allc else 1, "kind": "oracle",
        "sample": (f"decode GEMM of the Qwen3-8B block at M in {{1,4,16}}: the first {args.cpu_rows} output rows of "
                   f"each of the 7 projections per job, one job on 1 core and one job per core on {cores} spawned "
                   f"processes (os.sched_getaffinity) started together; quantize+pack: 64 rows of each projection per "
                   f"job; EAR/KL: 8 tokens x 151936 per job; GPTQ: one {GPTQ_SHAPES[0][0]} x {GPTQ_SHAPES[0][1]} layer with "
                   f"{GPTQ_SHAPES[0][2]} calibration rows at b = {GPTQ_SHAPES[0][3]} on one core (binary64 scalar C "
                   f"oracle, unchanged)"),
        "single_core": {"gemm_GBps": r(rates["gemm_1core"]), "quantize_GBps": r(rates["quantize_1core"]),
                        "ear_kl_GBps": r(rates["ear_1core"]), "gptq_s_per_layer": r(rates["gptq_1core_s"])},
        "all_cores": None if not allc else {"cores": cores, "gemm_GBps": r(rates["gemm_allcore"]),
                                            "quantize_GBps": r(rates["quantize_allcore"]),
                                            "ear_kl_GBps": r(rates["ear_allcore"])},
        "wall_s": round(rates["wall_s"], 1),
    }


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cores = _host_cores()
    job = _gemm_job(args.cpu_rows)
    for _ in range(args.warmup):
        _run_parallel([job] * cores)
    nbytes, span = 0, 0.0
    for _ in range(args.steps):
        nb, sp = _run_parallel([job] * cores)
        nbytes += nb
        span += sp
    value = nbytes / span / 1e9
    sample = (f"first {args.cpu_rows} output rows of each of the 7 Qwen3-8B-block projections, M in {{1,4,16}}, "
              f"one job per core on {cores} spawned processes started together (binary64 scalar C oracle); "
              "each step one job per core")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(span / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "block_weight_bytes": BLOCK_BYTES, "bytes_per_step": 3 * BLOCK_BYTES,
                   "parallelism": "rank 0 alone, on the host cores",
                   "sample": f"first {args.cpu_rows} output rows of each projection per job (rows are independent)"},
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def decode_traffic():
    """DRAM bytes per decode launch of this workload from the committed ncu
    capture (profiles/decode_block_traffic.txt), or None when the kernel
    source has changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "decode_block_traffic.txt")
    src = os.path.join(ROOT, "weight_only_mixed_b200", "csrc", "gemm_decode.cu")
    try:
        with open(path) as f:
            rec = json.load(f)
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    if rec.get("gemm_decode_cu_sha256") != sha:
        return None
    return rec.get("dram_bytes_per_launch")


def run_case(args):
    """One kernel of the path, launched on its own (for ncu captures)."""
    import torch
    import synth
    import weight_only_mixed_b200 as slq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    kind, *parts = args.case.split(":")
    vals = [float(p) if "." in p else int(p) for p in parts]
    if kind == "block":
        calls = []
        for M in DECODE_MS:
            qws = [slq.quantize(synth.weights_torch(N, K, seed=synth.SEED_WEIGHTS + 10 * i, device=dev), b)
                   for i, (_, N, K, b) in enumerate(QWEN3_8B_BLOCK)]
            xs = [synth.activations_torch(M, K, seed=synth.SEED_X + 10 * i + M, device=dev)
                  for i, (_, N, K, b) in enumerate(QWEN3_8B_BLOCK)]
            for grp in BLOCK_LAUNCHES:
                calls.append([(xs[i], qws[i]) for i in grp])

        def fn():
            for items in calls:
                if len(items) == 1:
                    slq.gemm(items[0][0], items[0][1], stream=stream)
                else:
                    slq.gemm_group(items, stream=stream)
        per_call = len(calls)
    elif kind in ("gemv", "decode", "tiled"):
        N, K, b, M = vals
        # Enough weight copies that consecutive calls miss in L2 (256 MB total).
        W0 = synth.weights_torch(N, K, device=dev)
        nrot = max(1, -(-(256 << 20) // weight_bytes(N, K, b)))
        qws = [slq.quantize(W0, b)] + [slq.quantize(W0 * (1.0 + 2.0**-7 * r), b) for r in range(1, nrot)]
        del W0
        x = synth.activations_torch(M, K, device=dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        it = [0]

        def fn():
            slq.gemm(x, qws[it[0] % nrot], out=y, path=kind, stream=stream)
            it[0] += 1
        per_call = 1
    elif kind == "ear":
        T, V, tau = vals
        a, bq = synth.logits_torch(T, V, device=dev)

        def fn():
            slq.ear_kl(a, bq, float(tau), stream=stream)
        per_call = 2  # the reduction and the token means
    elif kind == "eartopk":
        T, V, tau, k = vals
        a, bq = synth.logits_torch(T, V, device=dev)

        def fn():
            slq.ear_kl(a, bq, float(tau), top_k=int(k), stream=stream)
        per_call = 2
    elif kind == "quantize":
        N, K, b = vals
        W = synth.weights_torch(N, K, device=dev)
        q = slq.empty_quantized(N, K, b, dev)

        def fn():
            slq.quantize(W, b, out=q, stream=stream)
        per_call = 1
    elif kind == "gptq":
        N, K, T, b = vals
        W = synth.weights_torch(N, K, device=dev)
        X = torch.from_numpy(synth.calibration(T, K).view(np.int16)).to(dev).view(torch.bfloat16)
        out = slq.empty_quantized(N, K, b, dev)
        ws = torch.empty(slq.gptq_workspace_bytes(N, K), dtype=torch.uint8, device=dev)

        def fn():
            slq.gptq(W, X, b, out=out, workspace=ws, stream=stream)
        per_call = 6 * (K // 32) + 2 * (K // 128) + 3
    elif kind == "gridnoise":
        N, K, b = vals
        W = synth.weights_torch(N, K, device=dev)

        def fn():
            slq.grid_noise(W, b, stream=stream)
        per_call = 1
    else:
        raise SystemExit(f"unknown --case {args.case}")
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    run = fn
    if args.graph:
        # The calls captured in one CUDA graph: device time without the
        # host's per-call cost (small layers take less than a Python call).
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(args.steps):
                fn()
        graph.replay()
        torch.cuda.synchronize()
        run = graph.replay
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if args.graph:
        run()
    else:
        for _ in range(args.steps):
            run()
    e1.record(stream)
    e1.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / max(1, args.steps)
    print(json.dumps({"case": args.case, "avg_us_per_call": round(us, 3), "launches_per_call": per_call,
                      "calls": args.steps, "warmup": args.warmup, "graph": bool(args.graph)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["slq", "reference"], default="slq")
    ap.add_argument("--repeat", type=int, default=1, help="graph replays per counted step group")
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=128,
                    help="output rows of each projection in the oracle's GEMM sample")
    ap.add_argument("--cpu-single", action="store_true", help="cpu_baseline on one core only")
    ap.add_argument("--case", default=None, help="run one kernel on its own (see the module docstring)")
    ap.add_argument("--graph", action="store_true", help="--case: time the calls as one captured CUDA graph")
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_slq(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
