"""Benchmark of the GEMM library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {smgemm,reference}] [--headline-only]

One step is one call of the hot path on one batch of synthetic input. The headline
workload is the square BF16 GEMM (A[4096,4096] row-major x B[4096,4096] column-major,
FP32 accumulation, BF16 out); its throughput in TFLOP/s is ``value``. The other
workloads (tiny FP16, the FFN pair and the backward GEMMs of its first layer, eight
grouped GEMMs in one launch and as eight calls, FP8 block-scaled GEMM and its
quantiser, the LM-head GEMM at M in {1,4,16,64} and, at M = 16, fused with the row
log-softmax) are timed the same way and reported under ``configs``. FLOPs are 2*M*N*K; bytes count every operand once.

Timing: W untimed warm-up steps, then K steps between CUDA events on the launching
stream, bracketed by a barrier and a device synchronise; the maximum over ranks is
taken. Workloads whose operands fit in L2 rotate over enough copies that the bytes
touched between two uses of one copy exceed L2. SM clocks and throttle reasons are
read through NVML over and over while the headline's timed calls run (and by nvidia-smi
every 200 ms over the same window). After that region the
headline also times at least 50 further calls one by one (events around each call) and
reports their median, minimum and maximum.

``--impl reference`` times the CPU oracle (plain FP64 triple loop) on a bounded
sample of the same workload on the host cores, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "GEMM TFLOPS & % of B200 tensor peak (BF16/FP8); GB/s & % HBM for skinny M"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Sources of the headline kernel (gemm_tc16_pair_kernel): a recorded DRAM-traffic figure
# is only reported while these are unchanged since its ncu capture.
KERNEL_SOURCES = ["sm_gemm_b200/csrc/gemm_tc16_pair.cu", "sm_gemm_b200/csrc/operands.cuh",
                  "sm_gemm_b200/csrc/sm100.cuh", "sm_gemm_b200/csrc/epilogue.cuh",
                  "sm_gemm_b200/csrc/fp8_codec.cuh", "sm_gemm_b200/csrc/kernels.h"]


# ----------------------------------------------------------------------------- utilities

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d[kernel][workload]
        if e.get("source_hash") != kernel_source_hash():
            return None
        return float(e["dram_bytes_per_launch"])
    except (KeyError, ValueError, TypeError):
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while active."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


class NvmlClocks:
    """The SM clock and the active clock-event (throttle) reasons read in-process through
    NVML (what nvidia-smi reports), so that they can be sampled many times within a timed
    region of a few milliseconds, shorter than nvidia-smi's sampling period. Reading only:
    no setting of the GPU is touched."""

    def __init__(self, uuid):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.names = [(getattr(pynvml, "nvmlClocksEventReasonHwSlowdown", 0x8), "hw_slowdown"),
                          (getattr(pynvml, "nvmlClocksEventReasonHwThermalSlowdown", 0x40), "hw_thermal_slowdown"),
                          (getattr(pynvml, "nvmlClocksEventReasonSwThermalSlowdown", 0x20), "sw_thermal_slowdown"),
                          (getattr(pynvml, "nvmlClocksEventReasonSwPowerCap", 0x4), "sw_power_cap")]
            self.ok = True
        except Exception:
            self.ok = False

    def sample(self):
        if not self.ok:
            return
        try:
            self.samples.append((float(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)),
                                 int(self.get_reasons(self.h))))
        except Exception:
            self.ok = False

    # A background thread reads back to back from begin() to end() (NVML calls run
    # outside the interpreter lock, so the launching thread is not held up).
    def begin(self):
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def _run(self):
        while not self._stop.is_set() and self.ok:
            self.sample()

    def end(self):
        self._stop.set()
        self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return None
        reasons = sorted({n for _, r in self.samples for bit, n in self.names if r & bit})
        return {"sm_mhz": float(np.median([m for m, _ in self.samples])), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml, during the timed region"}


def merge_clocks(nvml_summary, smi_summary):
    """The clock record of the JSON line: NVML samples taken while the timed calls ran
    when there are any, with nvidia-smi's samples (every 200 ms over the same window,
    often none within a region of a few milliseconds) beside them; else nvidia-smi's."""
    if nvml_summary is None:
        return dict(smi_summary, source="nvidia-smi")
    out = dict(nvml_summary)
    out["nvidia_smi"] = smi_summary
    if smi_summary.get("sm_max_mhz"):
        out["sm_max_mhz"] = smi_summary["sm_max_mhz"]
    out["reasons"] = sorted(set(out["reasons"]) | set(smi_summary.get("reasons", [])))
    return out


# ----------------------------------------------------------------------------- GPU arm

# About 50 us of SM cycles: enough for the host to queue a few calls ahead.
QUEUE_AHEAD_CYCLES = 100_000
# Shortest timed region for the per-workload lines (see Ctx.time).
MIN_TIMED_MS = 2.0
# Device warm-up before the headline's own warm-up steps: ~50 ms of a spin kernel. The
# first timed region of a process otherwise ran 0.5-3 us per call slower than the next
# ones on the same data (measured on B200 boxes; with the spin the difference was gone).
DEVICE_WARMUP_CYCLES = 100_000_000


def time_steps(torch, step, warmup: int, steps: int, dist=None, during=None):
    """Device time of `steps` calls of step(i) after `warmup` calls: CUDA events on the
    current stream, barrier + synchronise on both sides, max over ranks (ms total).

    A short spin kernel runs before the start event: while the device is busy with it
    the host queues the first timed calls, so the timed region starts with work queued
    instead of with the device waiting for the first launch to come through. `during`
    (optional) has begin() called just before the start event and end() once the end
    event has completed (clock sampling over the timed region)."""
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    if during is not None:
        during.begin()
    torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
    s.record()
    for i in range(steps):
        step(warmup + i)
    e.record()
    torch.cuda.synchronize()
    if during is not None:
        during.end()
    if dist is not None:
        dist.barrier()
    return max_over_ranks(s.elapsed_time(e), dist)


def graph_us_per_call(torch, step, calls: int, replays: int = 3) -> float:
    """Device time per call (us) of `calls` consecutive calls of step(i) captured in one
    CUDA graph and replayed (best of `replays` timed replays): the calls' own device time
    back to back, without the host's per-call cost, which paces kernels of a few
    microseconds when a Python loop launches them one by one."""
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(0)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for i in range(calls):
            step(i)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(replays):
        graph.replay()
        torch.cuda.synchronize()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
        s.record()
        graph.replay()
        e.record()
        torch.cuda.synchronize()
        best = min(best, s.elapsed_time(e) * 1e3 / calls)
    del graph
    return round(best, 2)


def per_call_us(torch, step, start: int, calls: int) -> dict:
    """Median, min and max device time (us) of `calls` further calls of step(i), each
    bracketed by its own CUDA events on the current stream (run after the timed region,
    so its events do not touch the headline timing)."""
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(calls + 1)]
    step(start)  # not measured: keeps the device busy while the measured calls are queued
    ev[0].record()
    for i in range(calls):
        step(start + 1 + i)
        ev[i + 1].record()
    torch.cuda.synchronize()
    return call_stats([ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(calls)])


def call_stats(us) -> dict:
    t = sorted(us)
    n = len(t)
    med = t[n // 2] if n % 2 else 0.5 * (t[n // 2 - 1] + t[n // 2])
    return {"median": round(med, 2), "min": round(t[0], 2), "max": round(t[-1], 2), "calls": n}


def max_over_ranks(x: float, dist=None) -> float:
    """The largest of every rank's x (all ranks call it; NCCL reduces on the device,
    other backends on the host)."""
    if dist is None:
        return x
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step: float, steps: int, world: int, ms_total: float) -> float:
    """Aggregate throughput of `world` replicas that each ran `steps` steps of
    `flops_per_step` in at most `ms_total` milliseconds (the slowest rank's time)."""
    return flops_per_step * steps * world / (ms_total / 1e3) / 1e12


def n_copies(bytes_per_set: int) -> int:
    return max(1, -(-2 * L2_BYTES // max(bytes_per_set, 1)) + 1) if bytes_per_set < 2 * L2_BYTES else 1


class Ctx:
    def __init__(self, args, world, dist):
        import torch
        import sm_gemm_b200 as sg
        import synth
        from sm_gemm_b200 import metrics
        self.torch, self.sg, self.synth, self.metrics = torch, sg, synth, metrics
        self.dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
        torch.cuda.set_device(self.dev)
        self.peaks = load_peaks()
        self.fp8_peak = 2.0 * self.peaks["bf16_tflops"]   # measured bf16 x nominal fp8/bf16 ratio (2)
        self.W, self.K = args.warmup, args.steps
        self.min_ms = args.min_timed_ms if args.min_timed_ms > 0 else None
        self.world, self.dist = world, dist
        self.launches = 0
        self.results = {}

    def time(self, step, launches_per_step=1, warmup=None, steps=None, min_ms="default", during=None):
        """Device time (ms) of K calls of step. With min_ms (and no explicit step
        count), a workload whose K calls took less than min_ms is timed again over
        enough calls to span it, and the result is scaled back to K calls: kernels of a
        few microseconds are then not measured over a region as short as their launch
        jitter. The headline passes min_ms=None and is timed over exactly K steps."""
        w = self.W if warmup is None else warmup
        k = self.K if steps is None else steps
        if min_ms == "default":
            min_ms = self.min_ms
        ms = time_steps(self.torch, step, w, k, self.dist, during=during)
        self.launches += launches_per_step * k
        if steps is None and min_ms is not None and 0 < ms < min_ms:
            k2 = int(math.ceil(k * min_ms / ms))
            ms2 = time_steps(self.torch, step, 0, k2, self.dist)
            self.launches += launches_per_step * k2
            ms = ms2 * k / k2
        return ms

    def record(self, name, ms_total, steps, flops=None, nbytes=None, peak_tf=None, extra=None):
        t = ms_total / steps / 1e3
        r = {"us_per_call": round(t * 1e6, 2)}
        if flops is not None:
            r["tflops"] = round(flops / t / 1e12, 1)
            if peak_tf:
                r["frac_tensor_peak"] = round(flops / t / 1e12 / peak_tf, 4)
        if nbytes is not None:
            r["gbs"] = round(nbytes / t / 1e9, 1)
            r["frac_hbm"] = round(nbytes / t / 1e9 / self.peaks["hbm_gbs"], 4)
        if extra:
            r.update(extra)
        self.results[name] = r
        return r

    def t(self, x, dtype=None):
        return self.torch.from_numpy(np.ascontiguousarray(x)).to(dtype or self.torch.bfloat16).to(self.dev)


def wl_square_bf16(c: Ctx, headline: bool):
    """Square BF16 4096^3 (the headline): returns the JSON line's core fields."""
    torch, sg, m = c.torch, c.sg, c.metrics
    n = 4096
    d = c.synth.square_bf16(n)
    A0, Bt0 = c.t(d["A"]), c.t(d["Bt"])
    set_bytes = m.gemm_bytes(n, n, n, "bf16", "bf16", "bf16")
    copies = n_copies(set_bytes)
    As = [A0] + [A0.clone() for _ in range(copies - 1)]
    Bs = [Bt0] + [Bt0.clone() for _ in range(copies - 1)]
    Cs = [torch.empty((n, n), dtype=torch.bfloat16, device=c.dev) for _ in range(copies)]
    ws = torch.empty(max(sg.workspace_size(n, n, n, 0), 16), dtype=torch.uint8, device=c.dev)

    def step(i):
        j = i % copies
        sg.gemm_bf16(As[j], Bs[j].t(), out=Cs[j], workspace=ws)

    torch.cuda._sleep(DEVICE_WARMUP_CYCLES)
    torch.cuda.synchronize()
    try:
        smi_id = "GPU-" + str(torch.cuda.get_device_properties(c.dev).uuid)
    except Exception:
        smi_id = str(c.dev.index)
    nvml = NvmlClocks(smi_id)
    with ClockSampler(smi_id) as clk:
        ms = c.time(step, min_ms=None, during=nvml if nvml.ok else None)
    dist_us = per_call_us(torch, step, c.W + c.K, max(50, c.K))
    assert sg.check() == sg.OK
    flops = m.gemm_flops(n, n, n)
    plan = sg.last_config()
    c.record("square_bf16_4096", ms, c.K, flops=flops, peak_tf=c.peaks["bf16_tflops"],
             extra={"plan": plan, "per_call_us": dist_us})
    out = {"ms": ms, "flops": flops, "copies": copies, "set_bytes": set_bytes, "plan": plan,
           "clocks": merge_clocks(nvml.summary(), clk.summary())}
    if not headline:
        return out
    # End to end through the public API from pinned host buffers: every step uploads its
    # A and B and downloads its C. Steps are pipelined over two device buffer sets: the
    # upload of step i+1 (one stream) and the download of step i-1 (another) overlap the
    # GEMM of step i (a third), so PCIe runs in both directions while the tensor cores
    # work. The timing stream only records the start/end events and waits for every
    # download, so the timed region covers all copies.
    Ah = torch.from_numpy(np.ascontiguousarray(d["A"])).to(torch.bfloat16).pin_memory()
    Bh = torch.from_numpy(np.ascontiguousarray(d["Bt"])).to(torch.bfloat16).pin_memory()
    Chs = [torch.empty((n, n), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    Ads = [torch.empty_like(A0) for _ in range(2)]
    Bds = [torch.empty_like(Bt0) for _ in range(2)]
    Cds = [torch.empty_like(Cs[0]) for _ in range(2)]
    s_up, s_gemm, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("up", "gemm", "down")}
    used = {k: [False, False] for k in ev}

    e2e_warm = max(3, c.W)

    def e2e_step(i):
        j, timer = i % 2, torch.cuda.current_stream()
        with torch.cuda.stream(s_up):
            if i == e2e_warm:
                s_up.wait_stream(timer)                  # the first timed upload follows the start event
            if used["gemm"][j]:
                s_up.wait_event(ev["gemm"][j])           # the GEMM of step i-2 has read this set
            Ads[j].copy_(Ah, non_blocking=True)
            Bds[j].copy_(Bh, non_blocking=True)
            ev["up"][j].record(s_up)
        with torch.cuda.stream(s_gemm):
            s_gemm.wait_event(ev["up"][j])
            if used["down"][j]:
                s_gemm.wait_event(ev["down"][j])         # step i-2's result has left this buffer
            sg.gemm_bf16(Ads[j], Bds[j].t(), out=Cds[j], workspace=ws, stream=s_gemm)
            ev["gemm"][j].record(s_gemm)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev["gemm"][j])
            Chs[j].copy_(Cds[j], non_blocking=True)
            ev["down"][j].record(s_down)
        timer.wait_event(ev["down"][j])
        for k in used:
            used[k][j] = True

    # As many steps as the headline: the pipeline's fill (the first upload) and drain (the
    # last GEMM and download) are then spread over K steps, as in a long-running job.
    e2e_steps = max(4, c.K)
    e2e_ms = c.time(e2e_step, warmup=e2e_warm, steps=e2e_steps)
    out["e2e"] = {"value": round(whole_job_tflops(flops, e2e_steps, c.world, e2e_ms), 2), "unit": "TFLOP/s",
                  "h2d_bytes_per_step": 2 * n * n * 2, "d2h_bytes_per_step": n * n * 2}
    return out


def wl_tiny_fp16(c: Ctx):
    torch, sg = c.torch, c.sg
    t = c.synth.tiny_fp16()
    A, B = c.t(t["A"], torch.float16), c.t(t["B"], torch.float16)
    C = torch.empty((64, 64), dtype=torch.float32, device=c.dev)
    step = lambda i: sg.gemm_bf16(A, B, out=C)
    ms = c.time(step)
    plan = sg.last_config()
    g_us = graph_us_per_call(torch, step, max(c.K, 20))
    c.launches += 6 * max(c.K, 20) + 1  # warm-up call + 3 x (warm + timed) replays
    c.record("tiny_fp16_64", ms, c.K, flops=c.metrics.gemm_flops(64, 64, 64),
             extra={"plan": plan, "graph_us_per_call": g_us})


def wl_ffn(c: Ctx):
    torch, sg, m = c.torch, c.sg, c.metrics
    f = c.synth.ffn_pair()
    X, W1, W2, b1 = c.t(f["X"]), c.t(f["W1"]), c.t(f["W2"]), c.t(f["b1"])
    H = torch.empty((1024, 16384), dtype=torch.bfloat16, device=c.dev)
    Y = torch.empty((1024, 4096), dtype=torch.bfloat16, device=c.dev)
    ws = torch.empty(max(sg.workspace_size(1024, 16384, 4096), sg.workspace_size(1024, 4096, 16384), 16),
                     dtype=torch.uint8, device=c.dev)
    ws8 = torch.empty(max(sg.workspace_size(1024, 4096, 16384, 1), 16), dtype=torch.uint8, device=c.dev)
    ms1 = c.time(lambda i: sg.gemm_bf16(X, W1, bias=b1, act="gelu_tanh", out=H, workspace=ws))
    p1 = sg.last_config()
    ms2 = c.time(lambda i: sg.gemm_bf16(H, W2, out=Y, workspace=ws))
    p2 = sg.last_config()
    fl = m.gemm_flops(1024, 16384, 4096)
    pk = c.peaks["bf16_tflops"]
    c.record("ffn_gemm1_bias_gelu", ms1, c.K, flops=fl, peak_tf=pk, extra={"plan": p1})
    c.record("ffn_gemm2", ms2, c.K, flops=fl, peak_tf=pk, extra={"plan": p2})
    c.record("ffn_pair", ms1 + ms2, c.K, flops=2 * fl, peak_tf=pk)
    # The same layer with FP8 activations between the GEMMs: GEMM1's epilogue emits H as
    # E4M3 codes + 1x128 scales, GEMM2 is the block-scaled FP8 GEMM on them (W2 quantised
    # once, outside the timed region).
    Hq = torch.empty((1024, 16384), dtype=torch.uint8, device=c.dev)
    Hs = torch.empty((128, 1024), dtype=torch.float32, device=c.dev)
    W2q, W2s = sg.quantize_fp8_blockwise(c.t(f["W2"], torch.float32), 128)
    ms3 = c.time(lambda i: sg.gemm_bf16_fp8out(X, W1, bias=b1, act="gelu_tanh", Q=Hq, scales=Hs, workspace=ws))
    ms4 = c.time(lambda i: sg.gemm_fp8_blockscaled(Hq, Hs, W2q, W2s, out=Y, workspace=ws8))
    c.record("ffn_gemm1_bias_gelu_fp8out", ms3, c.K, flops=fl, peak_tf=pk)
    c.record("ffn_gemm2_fp8", ms4, c.K, flops=fl, peak_tf=c.fp8_peak)


def wl_ffn_backward(c: Ctx):
    """Backward GEMMs of the FFN's first layer through layout flags: dX = dH W1^T (W1 read
    as a column-major B) and dW1 = X^T dH (X read as a column-major A). Each call moves
    more than L2 (W1 is 128 MB; dW1 writes 128 MB)."""
    torch, sg, m = c.torch, c.sg, c.metrics
    f = c.synth.ffn_backward()
    X, W1, dH = c.t(f["X"]), c.t(f["W1"]), c.t(f["dH"])
    dX = torch.empty((1024, 4096), dtype=torch.bfloat16, device=c.dev)
    dW1 = torch.empty((4096, 16384), dtype=torch.bfloat16, device=c.dev)
    ws = torch.empty(max(sg.workspace_size(1024, 4096, 16384), sg.workspace_size(4096, 16384, 1024), 16),
                     dtype=torch.uint8, device=c.dev)
    ms1 = c.time(lambda i: sg.gemm_bf16(dH, W1.t(), out=dX, workspace=ws))
    p1 = sg.last_config()
    ms2 = c.time(lambda i: sg.gemm_bf16(X.t(), dH, out=dW1, workspace=ws))
    p2 = sg.last_config()
    fl = m.gemm_flops(1024, 4096, 16384)
    pk = c.peaks["bf16_tflops"]
    c.record("ffn_backward_dX", ms1, c.K, flops=fl, peak_tf=pk, extra={"plan": p1})
    c.record("ffn_backward_dW1", ms2, c.K, flops=fl, peak_tf=pk, extra={"plan": p2})


def wl_grouped(c: Ctx):
    """Eight independent GEMMs X_g[128(g+1), 4096] x W_g[4096, 4096] (4608 rows in all):
    one grouped launch against the same GEMMs issued one call each. W is 256 MB."""
    torch, sg, m = c.torch, c.sg, c.metrics
    d = c.synth.grouped_experts()
    Xs, Ws = [c.t(x) for x in d["X"]], [c.t(w) for w in d["W"]]
    Ys = [torch.empty((x.shape[0], 4096), dtype=torch.bfloat16, device=c.dev) for x in Xs]
    ws = torch.empty(max([sg.workspace_size(x.shape[0], 4096, 4096) for x in Xs] +
                         [int(sg.lib().smgemm_grouped_workspace_size(len(Xs))), 16]), dtype=torch.uint8, device=c.dev)
    fl = sum(m.gemm_flops(x.shape[0], 4096, 4096) for x in Xs)
    pk = c.peaks["bf16_tflops"]
    ms = c.time(lambda i: sg.gemm_bf16_grouped(Xs, Ws, outs=Ys, workspace=ws))
    plan = sg.last_config()

    def separate(i):
        for x, w, y in zip(Xs, Ws, Ys):
            sg.gemm_bf16(x, w, out=y, workspace=ws)
    ms_sep = c.time(separate, launches_per_step=len(Xs))
    c.record("grouped_experts_8x4096x4096", ms, c.K, flops=fl, peak_tf=pk, extra={"plan": plan})
    c.record("grouped_experts_8x4096x4096_as_8_calls", ms_sep, c.K, flops=fl, peak_tf=pk)


def wl_fp8(c: Ctx, quant=True, gemm=True):
    torch, sg, m = c.torch, c.sg, c.metrics
    f8 = c.synth.fp8_blockscaled()
    Af, Bf = c.t(f8["A"], torch.float32), c.t(f8["B"], torch.float32)
    qa = torch.empty((2048, 4096), dtype=torch.uint8, device=c.dev)
    sa = torch.empty((32, 2048), dtype=torch.float32, device=c.dev)
    qb = torch.empty((16384, 4096), dtype=torch.uint8, device=c.dev)
    sb = torch.empty((32, 128), dtype=torch.float32, device=c.dev)
    if quant:
        # A (32 MB in, 8 MB out) fits in L2: rotate copies so every call reads HBM.
        na = n_copies(m.quant_bytes(2048, 4096, 1))
        Afs = [Af] + [Af.clone() for _ in range(na - 1)]
        qas = [qa] + [torch.empty_like(qa) for _ in range(na - 1)]
        sas = [sa] + [torch.empty_like(sa) for _ in range(na - 1)]
        qstep = lambda i: sg.quantize_fp8_blockwise(Afs[i % na], 1, Q=qas[i % na], scales=sas[i % na])
        msa = c.time(qstep)
        ga_us = graph_us_per_call(torch, qstep, max(c.K, 20))
        c.launches += 6 * max(c.K, 20) + 1  # warm-up call + 3 x (warm + timed) replays
        del Afs, qas[1:], sas[1:]
        msb = c.time(lambda i: sg.quantize_fp8_blockwise(Bf, 128, Q=qb, scales=sb))
        c.record("quant_1x128_A_2048x4096", msa, c.K, nbytes=m.quant_bytes(2048, 4096, 1),
                 extra={"graph_us_per_call": ga_us})
        c.record("quant_128x128_B_4096x16384", msb, c.K, nbytes=m.quant_bytes(4096, 16384, 128))
    else:
        sg.quantize_fp8_blockwise(Af, 1, Q=qa, scales=sa)
        sg.quantize_fp8_blockwise(Bf, 128, Q=qb, scales=sb)
    del Af, Bf
    if not gemm:
        return
    set8 = m.fp8_gemm_bytes(2048, 16384, 4096, "bf16")
    n8 = n_copies(set8)
    qas = [qa] + [qa.clone() for _ in range(n8 - 1)]
    qbs = [qb] + [qb.clone() for _ in range(n8 - 1)]
    C8 = [torch.empty((2048, 16384), dtype=torch.bfloat16, device=c.dev) for _ in range(n8)]
    ws = torch.empty(max(sg.workspace_size(2048, 16384, 4096, 1), 16), dtype=torch.uint8, device=c.dev)
    ms = c.time(lambda i: sg.gemm_fp8_blockscaled(qas[i % n8], sa, qbs[i % n8], sb, out=C8[i % n8], workspace=ws))
    c.record("fp8_blockscaled_2048x16384x4096", ms, c.K, flops=m.gemm_flops(2048, 16384, 4096), peak_tf=c.fp8_peak,
             extra={"plan": sg.last_config(), "peak_note": "fp8 peak = 2 x measured bf16 (nominal ratio)"})


def wl_lm_head(c: Ctx, ms_list=(1, 4, 16, 64)):
    torch, sg, m = c.torch, c.sg, c.metrics
    Wl = c.t(c.synth.lm_head(m=1)["W"])
    ws = torch.empty(max(max(sg.workspace_size(mm, 128256, 4096) for mm in ms_list), 16), dtype=torch.uint8,
                     device=c.dev)
    for mm in ms_list:
        Xl = c.t(c.synth.lm_head(m=mm, vocab=8)["X"])
        Cl = torch.empty((mm, 128256), dtype=torch.float32, device=c.dev)
        ms = c.time(lambda i: sg.gemm_bf16(Xl, Wl, out=Cl, workspace=ws))
        c.record(f"lm_head_m{mm}", ms, c.K, flops=m.gemm_flops(mm, 128256, 4096),
                 nbytes=m.gemm_bytes(mm, 128256, 4096, "bf16", "bf16", "f32"), extra={"plan": sg.last_config()})
    # The same LM head fused with the row log-softmax (2 launches: GEMM with per-tile
    # max/sum partials, then the merge and in-place subtract). Bytes add the second pass's read
    # and write of the FP32 output.
    mm = 16
    Xl = c.t(c.synth.lm_head(m=mm, vocab=8)["X"])
    Cl = torch.empty((mm, 128256), dtype=torch.float32, device=c.dev)
    wsl = torch.empty(max(int(sg.lib().smgemm_logsoftmax_workspace_size(mm, 128256, 4096)), 16), dtype=torch.uint8,
                      device=c.dev)
    ms = c.time(lambda i: sg.gemm_bf16_logsoftmax(Xl, Wl, out=Cl, workspace=wsl), launches_per_step=2)
    c.record(f"lm_head_logsoftmax_m{mm}", ms, c.K, flops=m.gemm_flops(mm, 128256, 4096),
             nbytes=m.gemm_bytes(mm, 128256, 4096, "bf16", "bf16", "f32") + 2 * mm * 128256 * 4,
             extra={"plan": sg.last_config()})


def wl_lm_head_vocab_parallel(c: Ctx, mm: int = 16):
    """The LM head (M = 16, V = 128256) with its row log-softmax, its vocabulary split over
    the ranks (each streams only its slice of W): GEMM with (max, sum exp) partials on the
    slice, all-gather of the partials (NCCL), merge and subtract. Strong scaling: the whole
    job is one LM head whatever the rank count; GB/s counts the whole head's bytes."""
    torch, sg, m = c.torch, c.sg, c.metrics
    from sm_gemm_b200 import vocab_parallel as vp
    V, K = 128256, 4096
    rank = c.dist.get_rank() if c.dist is not None else 0
    c0, c1 = vp.shard_columns(V, c.world, rank)
    d = c.synth.lm_head(m=mm)
    Xl = c.t(d["X"])
    Ws = c.t(np.ascontiguousarray(d["W"][:, c0:c1]))
    del d
    Cl = torch.empty((mm, c1 - c0), dtype=torch.float32, device=c.dev)
    ws = torch.empty(max(sg.workspace_size(mm, max(c1 - c0, 1), K), 16), dtype=torch.uint8, device=c.dev)
    # our kernels per step: the skinny GEMM (its epilogue forms the partials) and the merge +
    # subtract; the all-gather is NCCL's and the padding of short slices torch's
    ms = c.time(lambda i: vp.lm_head_log_softmax(Xl, Ws, V, dist=c.dist, out=Cl, workspace=ws),
                launches_per_step=2)
    c.record(f"lm_head_logsoftmax_vocab_parallel_m{mm}", ms, c.K, flops=m.gemm_flops(mm, V, K),
             nbytes=m.gemm_bytes(mm, V, K, "bf16", "bf16", "f32") + 2 * mm * V * 4,
             extra={"ranks": c.world, "slice_columns": c1 - c0, "scaling": "strong",
                    "exchange": "all-gather of per-tile (max, sum exp) pairs" if c.world > 1 else "none"})


def run_gpu(args, rank: int, world: int, dist):
    c = Ctx(args, world, dist)
    if args.only is not None and args.only != "square_bf16":
        {"tiny_fp16": lambda: wl_tiny_fp16(c), "ffn": lambda: wl_ffn(c),
         "fp8": lambda: wl_fp8(c, quant=False), "quant": lambda: wl_fp8(c, gemm=False),
         "ffn_bwd": lambda: wl_ffn_backward(c), "grouped": lambda: wl_grouped(c),
         "lm_head": lambda: wl_lm_head(c), "lm_head_vp": lambda: wl_lm_head_vocab_parallel(c)}[args.only]()
        assert c.sg.check() == c.sg.OK
        return {"only": args.only, "steps": c.K, "warmup": c.W, "gpu_launches": c.launches, "configs": c.results}

    h = wl_square_bf16(c, headline=args.only is None)
    if args.only is None and not args.headline_only:
        wl_tiny_fp16(c)
        wl_ffn(c)
        wl_ffn_backward(c)
        wl_grouped(c)
        wl_fp8(c)
        wl_lm_head(c)
        wl_lm_head_vocab_parallel(c)
    assert c.sg.check() == c.sg.OK
    peaks = c.peaks
    per_launch_s = h["ms"] / c.K / 1e3
    achieved = h["flops"] / per_launch_s / 1e12
    line = {
        "metric": METRIC, "value": round(whole_job_tflops(h["flops"], c.K, world, h["ms"]), 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": c.K, "warmup": c.W, "ms_per_step": round(h["ms"] / c.K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "square_bf16_4096", "M": 4096, "N": 4096, "K": 4096,
                   "layout": "A row-major, B column-major (W^T stored K-contiguous)", "out": "bf16",
                   "accumulate": "fp32",
                   "l2": f"rotating {h['copies']} input/output sets ({h['copies'] * h['set_bytes'] / 2**20:.0f} MiB) "
                         f"so reuse distance exceeds L2",
                   "parallelism": f"replicas{world}" if world > 1 else "single-gpu", "plan": h["plan"],
                   "device_warmup": "~50 ms spin kernel before the warm-up steps"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "peak_kind": f"{peaks['source']} bf16 burst",
                     "traffic": recorded_traffic("gemm_tc16_pair", "square_bf16_4096"),
                     "algorithmic_bytes": h["set_bytes"], "algorithmic_flops": h["flops"],
                     "kernel": "gemm_tc16_pair_kernel<64,6,kOutTma> (CTA pairs, 256x256 tiles, TMA-store epilogue)"},
        "gpu_launches": c.launches,
        "clocks": h["clocks"],
        "configs": c.results,
    }
    if "e2e" in h:
        line["e2e"] = h["e2e"]
    return line


# ----------------------------------------------------------------------------- CPU oracle

def cpu_cores() -> int:
    if os.environ.get("OMP_NUM_THREADS"):
        return int(os.environ["OMP_NUM_THREADS"])
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


_SQUARE_BITS = {}


def _square_bits():
    """The square BF16 workload as raw bf16 bits (generated once per process)."""
    if not _SQUARE_BITS:
        import torch
        import synth
        d = synth.square_bf16(4096)
        for k in ("A", "Bt"):
            _SQUARE_BITS[k] = torch.from_numpy(d[k]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return _SQUARE_BITS["A"], _SQUARE_BITS["Bt"]


def oracle_sample(rows: int):
    """Oracle (FP64 triple loop) on `rows` full rows of the square BF16 workload.
    Returns (seconds, flops)."""
    import oracle
    n = 4096
    Afull, Bt = _square_bits()
    A = Afull[:rows]
    t0 = time.perf_counter()
    oracle.gemm(A, Bt.T, a_dtype=oracle.BF16, b_dtype=oracle.BF16, out_dtype=oracle.BF16)
    return time.perf_counter() - t0, 2 * rows * n * n


def cpu_baseline(target_s: float = 10.0):
    t, _ = oracle_sample(16)
    rows = int(min(4096, max(16, 16 * target_s / max(t, 1e-3))))
    t, fl = oracle_sample(rows)
    return {"value": round(fl / t / 1e12, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{rows} of 4096 output rows of the square BF16 4096^3 GEMM (FP64 accumulation), "
                      f"{t:.1f} s"}


def run_reference(args):
    """Reference arm: the CPU oracle, as it stands, timed on bounded samples."""
    t, _ = oracle_sample(8)
    rows = int(min(4096, max(8, 8 * 4.0 / max(t, 1e-3))))          # ~4 s per step
    for _ in range(args.warmup):
        oracle_sample(max(8, rows // 8))
    total, fl_total = 0.0, 0
    for _ in range(args.steps):
        t, fl = oracle_sample(rows)
        total += t
        fl_total += fl
    v = fl_total / total / 1e12
    cb = {"value": round(v, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
          "sample": f"{rows} of 4096 output rows of the square BF16 4096^3 GEMM per step"}
    return {"metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "square_bf16_4096", "M": 4096, "N": 4096, "K": 4096,
                       "sample_rows_per_step": rows},
            "cpu_baseline": cb,
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main

def launch_ranks(n: int) -> int:
    """`--gpus n` without a launcher: start n ranks of this same command, one per GPU, with
    torch.distributed.run on this node (rendezvous on 127.0.0.1), and return their exit
    status. Refuses (status 2) when fewer than n GPUs are visible: it never times fewer
    GPUs than asked for."""
    import socket
    import torch
    have = torch.cuda.device_count()
    if have < n:
        print(f"bench.py: --gpus {n} but only {have} GPU(s) visible", file=sys.stderr)
        return 2
    with socket.socket() as sck:
        sck.bind(("127.0.0.1", 0))
        port = sck.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="smgemm", choices=["smgemm", "reference"])
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--min-timed-ms", type=float, default=MIN_TIMED_MS,
                    help="shortest timed region of a per-workload line (0: exactly --steps calls, "
                         "for a fixed launch sequence under a profiler)")
    ap.add_argument("--only", default=None,
                    choices=["square_bf16", "tiny_fp16", "ffn", "ffn_bwd", "grouped", "fp8", "quant", "lm_head",
                             "lm_head_vp"],
                    help="time one workload and print its line (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl != "reference" and args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl != "reference" and world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        sys.exit(2)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    line = run_gpu(args, rank, world, dist)
    if rank == 0 and not args.no_cpu_baseline and args.only is None:
        line["cpu_baseline"] = cpu_baseline()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
