"""Benchmark of the LLM.int8() matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 175b]
                    [--no-decode] [--no-variants] [--no-configs] [--no-cpu-baseline]

Prints ONE JSON line.  The headline workload is the 175B-scale FFN matmul
(X 4096 x 12288, W 12288 x 49152, 24 seeded outlier columns, threshold 6.0):
throughput in int8 TOPS (2*M*N*K per forward, all K counted) with the
dominant kernel's roofline against the dense-int8 tensor peak.  Objects on the
same line:
  decode       the decode-shaped FFN up-projection (X 8 x 4096, W 4096 x 11008)
               in HBM GB/s against the measured copy bandwidth, measured on
               forwards back to back (the launch alone reported beside it);
  configs      the prefill FFN and the attention-QKV sweep (0, 12, 48, 123
               outlier columns and threshold = inf) in TOPS;
  grouped      the group-wise variant at the headline shape (groups of 1024
               and 128);
  decode_int4  the 4-bit weight-only product on the decode workload;
  block_codec  the block-wise 8-bit codec on a 201 MB fp32 vector.

One step = one whole forward (outlier detection, X quantisation, outlier weight
gather, int8 GEMM with fused dequantising epilogue and fp16 outlier product);
the weight is prepared once, outside the timed region.  Inputs are synthetic
and seeded (see int8_quantized_matmul_02_b200.synth).  The `e2e` key is the
same metric through the public call with host buffers (int8mm_forward_host:
pinned X copied in, Y copied back to pinned memory in row bands that overlap
the product), the copies inside the timed region.

Multi-GPU: the path is one GPU with no collective; --gpus N runs N
independent replicas (one process per GPU, torchrun), weak scaling, timed as
the max over ranks.

--impl reference times the CPU oracle (the plain C implementation under
oracle/) on this host's cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int8_quantized_matmul_02_b200 import synth  # noqa: E402

NOMINAL_INT8_TOPS = 4500.0      # B200 dense int8, nominal
NOMINAL_BF16_TFLOPS = 2250.0    # B200 dense bf16, nominal
INT8_PER_BF16 = NOMINAL_INT8_TOPS / NOMINAL_BF16_TFLOPS
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD_NAMES = {
    "tiny": "tiny 16x256x384",
    "decode": "decode-shaped FFN up-proj 8x4096x11008",
    "prefill": "prefill FFN 2048x8192x28672",
    "175b": "175B-scale FFN 4096x12288x49152",
}
for _n in (0, 12, 48, 123):
    WORKLOAD_NAMES[f"qkv_o{_n}"] = f"attention QKV projection 16384x12288x36864, {_n} outlier dims"
WORKLOAD_NAMES["qkv_inf"] = "attention QKV projection 16384x12288x36864, threshold=inf"


# ----------------------------------------------------------------------------- helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region.

    The sampler polls every 20 ms from a reader thread that stamps each line
    with the host clock. Entering waits until the first sample has arrived, so
    polling is live when timing starts; `mark()` brackets the timed region and
    `summary()` keeps the samples inside it (the two nearest ones when the
    region is shorter than two polling periods, and says so)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.samples = []          # (host time, line)
        self.region = None

    def _read(self):
        for line in self.proc.stdout:
            if line.strip():
                self.samples.append((time.perf_counter(), line))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.PERIOD_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t_end = time.perf_counter() + 3.0
        while not self.samples and time.perf_counter() < t_end and self.proc.poll() is None:
            time.sleep(0.005)
        self.t_enter = time.perf_counter()
        return self

    def mark(self, which: str):
        """Host time of the start ('start') or end ('end') of the timed region."""
        now = time.perf_counter()
        if which == "start":
            self.region = [now, None]
        else:
            self.region[1] = now

    def __exit__(self, *exc):
        if self.region is None:
            self.region = [self.t_enter if self.proc else 0.0, time.perf_counter()]
        elif self.region[1] is None:
            self.region[1] = time.perf_counter()
        if self.proc is not None:
            time.sleep(2.5 * self.PERIOD_MS / 1000.0)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.thread.join(timeout=5)
        return False

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        parsed = []
        for t, line in list(self.samples):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, smax = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            parsed.append((t, sm, smax, [n for n, v in zip(names, parts[4:8]) if v.lower() == "active"]))
        if not parsed or self.region is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        t0, t1 = self.region
        inside = [p for p in parsed if t0 <= p[0] <= t1]
        basis = "inside the timed region"
        if len(inside) < 2:
            mid = 0.5 * (t0 + t1)
            inside = sorted(parsed, key=lambda p: abs(p[0] - mid))[:2]
            basis = "the two samples nearest the timed region (shorter than two polling periods)"
        sms = [p[1] for p in inside]
        reasons = sorted({r for p in inside for r in p[3]})
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": inside[-1][2], "reasons": reasons,
                "samples": len(inside), "period_ms": self.PERIOD_MS, "region_ms": round(1000 * (t1 - t0), 1),
                "basis": basis}


KERNEL_SOURCES = {
    "k_gemm_int8_2sm": ("gemm2sm_sm100.cuh", "gemm_sm100.cuh", "sm100_ptx.cuh"),
    "k_gemm_int8_sm100": ("gemm_sm100.cuh", "sm100_ptx.cuh"),
    "k_decode_int8_sm100": ("decode_sm100.cuh", "sm100_ptx.cuh"),
}


def strip_comments(src: str) -> str:
    """C/C++ source with every run of whitespace and // or /* */ comments
    outside string and character literals reduced to one space (literals kept
    as they are), so that editing a comment or the layout does not count as a
    change of the kernel."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif c.isspace() or src.startswith("//", i) or src.startswith("/*", i):
            # a run of whitespace and comments becomes one space
            while i < n:
                if src[i].isspace():
                    i += 1
                elif src.startswith("//", i):
                    j = src.find("\n", i)
                    i = n if j < 0 else j
                elif src.startswith("/*", i):
                    j = src.find("*/", i + 2)
                    i = n if j < 0 else j + 2
                else:
                    break
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return "".join(out).strip()


def kernel_source_sha(kernel: str) -> str:
    """Hash of the code (comments stripped) of the files a kernel is compiled from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int8_quantized_matmul_02_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary
    (profiles/traffic.json), or None when the kernel's sources changed since
    the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_sha") != kernel_source_sha(kernel):
        return None
    return float(e["dram_bytes_per_launch"])


# ----------------------------------------------------------------------------- our arm

def event_pairs(n: int, stream):
    """n (start, stop) timing events, created on the device (torch creates an
    event lazily at its first record; the library records raw handles)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in evs:
        a.record(stream)
        b.record(stream)
    stream.synchronize()
    return evs


def algorithmic_bytes_decode(wl, n_o: int) -> float:
    """Minimum HBM bytes of one decode forward: Wq + ca + X + Y + the fp16
    weight rows of the outlier dims."""
    return wl.N * wl.K + wl.N * 4 + wl.M * wl.K * 2 + wl.M * wl.N * 2 + n_o * wl.N * 2


def run_gemm_workload(wl, steps: int, warmup: int, dev, rank: int, cap: int):
    import int8_quantized_matmul_02_b200 as i8

    X, W, cols = synth.make_inputs(wl)
    Xd = X.to(dev)
    w = i8.prepare_weight(W.to(dev), cols)
    del W
    ws = i8.Workspace(wl.M, wl.K, wl.N, cap, device=dev)
    Y = torch.empty(wl.M, wl.N, dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream(dev)
    evs = event_pairs(steps, stream)

    def step(ev=None):
        lib = i8.library()
        import ctypes
        from int8_quantized_matmul_02_b200 import _abi
        opts = _abi.ForwardOpts(0, None, 0, ctypes.c_void_p(ev[0].cuda_event) if ev else None,
                                ctypes.c_void_p(ev[1].cuda_event) if ev else None)
        _abi.check(lib.int8mm_forward_ex(ctypes.c_void_p(Xd.data_ptr()), wl.M, ctypes.byref(w.struct),
                                         float(wl.threshold), ws.max_outliers, ctypes.c_void_p(Y.data_ptr()),
                                         ctypes.c_void_p(ws.buf.data_ptr()), ws.nbytes, ctypes.byref(opts),
                                         ctypes.c_void_p(stream.cuda_stream)), "int8mm_forward_ex")

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    st, n_o = i8.device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        clk.mark("start")
        t0.record(stream)
        for i in range(steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark("end")
    barrier()
    total_ms = t0.elapsed_time(t1)
    kern_ms = [a.elapsed_time(b) for a, b in evs]
    st, n_o = i8.device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")
    return {"total_ms": total_ms, "kern_ms": kern_ms, "n_o": n_o, "clocks": clk.summary(), "w": w, "ws": ws,
            "X": X, "Xd": Xd, "Y": Y}


def run_e2e(wl, state, steps: int, dev):
    """Same metric through the public API with host buffers (the package's
    forward() with a pinned CPU X and a pinned CPU Y, which calls
    int8mm_forward_host): X copied in, Y copied back in row bands overlapping
    the product, every copy inside the timed region."""
    import int8_quantized_matmul_02_b200 as i8

    Xh = state["X"].pin_memory()
    Yh = torch.empty(wl.M, wl.N, dtype=torch.float16, pin_memory=True)
    w, ws = state["w"], state["ws"]
    stream = torch.cuda.current_stream(dev)
    i8.forward(Xh, w, wl.threshold, workspace=ws, out=Yh)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        i8.forward(Xh, w, wl.threshold, workspace=ws, out=Yh)
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / steps
    return ms, wl.M * wl.K * 2, wl.M * wl.N * 2


def run_decode(steps: int, warmup: int, dev, cap: int, copies: int = 8):
    """Decode-shaped forward, rotating `copies` prepared weights so that the
    weights read between two uses of one copy exceed the 126 MB L2."""
    import ctypes

    import int8_quantized_matmul_02_b200 as i8
    from int8_quantized_matmul_02_b200 import _abi

    wl = synth.WORKLOADS["decode"]
    X, W, cols = synth.make_inputs(wl)
    Xd = X.to(dev)
    Wd = W.to(dev)
    ws_list, weights = [], []
    for c in range(copies):
        weights.append(i8.prepare_weight(Wd, cols))
        ws_list.append(i8.Workspace(wl.M, wl.K, wl.N, cap, device=dev))
    del Wd
    Y = torch.empty(wl.M, wl.N, dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream(dev)
    lib = i8.library()

    def fwd(i, ev=None):
        w = weights[i % copies]
        ws = ws_list[i % copies]
        opts = _abi.ForwardOpts(0, None, 0, ctypes.c_void_p(ev[0].cuda_event) if ev else None,
                                ctypes.c_void_p(ev[1].cuda_event) if ev else None)
        _abi.check(lib.int8mm_forward_ex(ctypes.c_void_p(Xd.data_ptr()), wl.M, ctypes.byref(w.struct),
                                         float(wl.threshold), ws.max_outliers, ctypes.c_void_p(Y.data_ptr()),
                                         ctypes.c_void_p(ws.buf.data_ptr()), ws.nbytes, ctypes.byref(opts),
                                         ctypes.c_void_p(stream.cuda_stream)), "int8mm_forward_ex")

    for i in range(max(warmup, copies)):
        fwd(i)
    torch.cuda.synchronize(dev)
    st, n_o = i8.device_status(ws_list[0])
    if st != 0:
        raise RuntimeError(f"decode device status {st}")
    # (1) kernel-only timing: events around the fused kernel of every step
    evs = event_pairs(steps, stream)
    for i in range(steps):
        fwd(i, evs[i])
    torch.cuda.synchronize(dev)
    kern_us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3
    # (2) back-to-back forwards, plain launches
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        fwd(i)
    b.record(stream)
    torch.cuda.synchronize(dev)
    plain_us = a.elapsed_time(b) * 1e3 / steps
    # (3) the same sequence captured once in a CUDA graph
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(copies * 4):
            fwd(i)
    g.replay()
    torch.cuda.synchronize(dev)
    reps = max(1, steps // (copies * 4))
    a.record(stream)
    for _ in range(reps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize(dev)
    graph_us = a.elapsed_time(b) * 1e3 / (reps * copies * 4)
    del g
    for ws in ws_list:
        st, _ = i8.device_status(ws)
        if st != 0:
            raise RuntimeError(f"decode device status {st} after timing")
    bytes_ = algorithmic_bytes_decode(wl, n_o)
    return {"wl": wl, "n_o": n_o, "kern_us": kern_us, "plain_us": plain_us, "graph_us": graph_us, "bytes": bytes_}


def algorithmic_bytes_int4(M: int, K: int, N: int, G: int) -> float:
    """Minimum HBM bytes of one 4-bit forward: packed codes + group constants + X + Y."""
    return N * K / 2 + N * (K // G) * 4 + M * K * 2 + M * N * 2


def run_int4_decode(steps: int, warmup: int, dev, G: int, copies: int = 8):
    """4-bit weight-only product on the decode workload's X and W, rotating
    `copies` prepared weights (8 x 22.5 MB > 126 MB L2).  Back-to-back calls
    (programmatic dependent launch) and the call alone (events around it)."""
    import int8_quantized_matmul_02_b200 as i8

    wl = synth.WORKLOADS["decode"]
    X, W, _ = synth.make_inputs(wl)
    Xd = X.to(dev)
    Wd = W.to(dev)
    weights = [i8.prepare_weight_int4(Wd, G) for _ in range(copies)]
    del Wd
    Y = torch.empty(wl.M, wl.N, dtype=torch.float16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for i in range(max(warmup, copies)):
        i8.forward_int4(Xd, weights[i % copies], out=Y, status=status, stream=stream)
    torch.cuda.synchronize(dev)
    evs = event_pairs(min(steps, 400), stream)
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        i8.forward_int4(Xd, weights[i % copies], out=Y, status=status, stream=stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    alone_us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        i8.forward_int4(Xd, weights[i % copies], out=Y, status=status, stream=stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    step_us = a.elapsed_time(b) * 1e3 / steps
    if int(status.item()) != 0:
        raise RuntimeError(f"int4 device status {int(status.item())}")
    return {"wl": wl, "G": G, "step_us": step_us, "alone_us": alone_us,
            "bytes": algorithmic_bytes_int4(wl.M, wl.K, wl.N, G)}


def run_codec(steps: int, warmup: int, dev):
    """Block-wise 8-bit codec of a 201 MB fp32 vector (larger than L2): quantise
    and dequantise, each timed with events over `steps` calls."""
    import int8_quantized_matmul_02_b200 as i8

    n, B = synth.CODEC_N, synth.CODEC_BLOCK
    x = synth.make_codec_vector().to(dev)
    q = torch.empty(n, dtype=torch.int8, device=dev)
    amax = torch.empty((n + B - 1) // B, dtype=torch.float32, device=dev)
    out = torch.empty(n, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        i8.block_quantize(x, B, q, amax, stream=stream)
        i8.block_dequantize(q, amax, B, out, stream=stream)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    c = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        i8.block_quantize(x, B, q, amax, stream=stream)
    b.record(stream)
    for _ in range(steps):
        i8.block_dequantize(q, amax, B, out, stream=stream)
    c.record(stream)
    torch.cuda.synchronize(dev)
    tq = a.elapsed_time(b) * 1e-3 / steps
    td = b.elapsed_time(c) * 1e-3 / steps
    nb = (n + B - 1) // B
    return {"n": n, "B": B, "quant_s": tq, "dequant_s": td,
            "quant_bytes": 4.0 * n + n + 4.0 * nb, "dequant_bytes": 1.0 * n + 4.0 * nb + 4.0 * n}


def run_grouped(wl, G: int, steps: int, warmup: int, dev, cap: int):
    """Group-wise forward (one constant per row/column and group of G
    consecutive k) on a large-M workload; the SM-pair GEMM kernel timed by
    events the library records around it."""
    import ctypes

    import int8_quantized_matmul_02_b200 as i8
    from int8_quantized_matmul_02_b200 import _abi

    X, W, cols = synth.make_inputs(wl)
    Xd = X.to(dev)
    w = i8.prepare_weight_grouped(W.to(dev), G, cols)
    del W
    ws = i8.Workspace(wl.M, wl.K, wl.N, cap, device=dev, G=G)
    Y = torch.empty(wl.M, wl.N, dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream(dev)
    lib = i8.library()
    evs = event_pairs(steps, stream)

    def step(ev=None):
        opts = _abi.ForwardOpts(0, None, 0, ctypes.c_void_p(ev[0].cuda_event) if ev else None,
                                ctypes.c_void_p(ev[1].cuda_event) if ev else None)
        _abi.check(lib.int8mm_forward_grouped(ctypes.c_void_p(Xd.data_ptr()), wl.M, ctypes.byref(w.struct),
                                              float(wl.threshold), ws.max_outliers, ctypes.c_void_p(Y.data_ptr()),
                                              ctypes.c_void_p(ws.buf.data_ptr()), ws.nbytes, ctypes.byref(opts),
                                              ctypes.c_void_p(stream.cuda_stream)), "int8mm_forward_grouped")

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        clk.mark("start")
        a.record(stream)
        for i in range(steps):
            step(evs[i])
        b.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark("end")
    st, n_o = i8.device_status(ws)
    if st != 0:
        raise RuntimeError(f"grouped device status {st}")
    return {"total_ms": a.elapsed_time(b), "kern_ms": [x.elapsed_time(y) for x, y in evs], "n_o": n_o,
            "clocks": clk.summary()}


_pg = None


def barrier():
    if _pg is not None:
        torch.distributed.barrier()


def combine_ranks(per_step_s: float, units_per_step: float, dev, distributed: bool):
    """Replicas: every rank times its own steps; the job's step time is the
    slowest rank's and the job's throughput is all ranks' units over it.
    Returns (max step seconds, job units per second)."""
    if not distributed:
        return per_step_s, units_per_step / per_step_s
    t = torch.tensor([per_step_s, units_per_step], dtype=torch.float64, device=dev)
    mx = t[:1].clone()
    torch.distributed.all_reduce(mx, op=torch.distributed.ReduceOp.MAX)
    tot = t[1:].clone()
    torch.distributed.all_reduce(tot, op=torch.distributed.ReduceOp.SUM)
    return float(mx.item()), float(tot.item()) / float(mx.item())


# ----------------------------------------------------------------------------- CPU oracle timing

def time_oracle_sample(wl, target_s: float = 12.0):
    """The CPU oracle, as it stands, on a bounded sample of the workload:
    outlier detection and quantisation of the whole X (timed in full), then the
    int8 product, outlier product and epilogue for the first n_cols columns of
    W, n_cols sized so the whole sample takes about target_s.  The weight
    conversion is one-time and excluded.  The product time grows linearly in
    the columns (each column is an independent dot product per row), so the
    whole forward's time is extrapolated as t_x + t_cols * N / n_cols and the
    throughput is 2 M N K over it: the figure does not depend on the sample
    size.  Returns (TOPS, seconds of the sample, cores, sample description)."""
    import oracle

    cores = oracle.default_threads()
    X, W, cols = synth.make_inputs(wl)
    Xn = X.numpy()

    def one(n_cols):
        prep = oracle.prepare_weight(W[:, :n_cols].contiguous().numpy(), cols)
        t0 = time.perf_counter()
        steps = oracle.forward_steps_abc(Xn, prep, wl.threshold)
        t1 = time.perf_counter()
        acc = oracle.int8_gemm(steps["xq"], prep["wq"], threads=cores)
        o = oracle.outlier_gemm(steps["xo"], steps["wo"])
        oracle.epilogue(acc, steps["ra"], prep["ca"], o)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1

    # calibrate the column slice with a 16-column probe
    t_x, t_p = one(16)
    per_col = t_p / 16
    n_cols = int(max(16, min(wl.N, (target_s - t_x) / max(per_col, 1e-9))))
    n_cols = n_cols // 16 * 16
    t_x, t_p = one(n_cols)
    t_full = t_x + t_p * wl.N / n_cols
    sample = (f"all {wl.M} rows of X through outlier detection and quantisation ({t_x:.2f} s), then the int8 "
              f"product, fp16 outlier product and epilogue for the first {n_cols} of {wl.N} output columns "
              f"({t_p:.2f} s); whole forward extrapolated as {t_x:.2f} + {t_p:.2f} x {wl.N}/{n_cols} s; weight "
              f"conversion excluded")
    return wl.ops / t_full / 1e12, t_x + t_p, cores, sample


# ----------------------------------------------------------------------------- main

def main():
    global _pg
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="175b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--max-outliers", type=int, default=1024)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=2000)
    ap.add_argument("--no-variants", action="store_true", help="skip the 4-bit and codec objects")
    ap.add_argument("--no-configs", action="store_true", help="skip the prefill and QKV-sweep objects")
    ap.add_argument("--only", choices=["decode", "decode_int4", "block_codec", "grouped"],
                    help="run one object alone (for profiling) and print it as the JSON line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world, rank, local = dist_info()
    wl = synth.WORKLOADS[args.workload]
    cfg = {"workload": WORKLOAD_NAMES[args.workload], "M": wl.M, "K": wl.K, "N": wl.N,
           "threshold": wl.threshold, "seeded_outlier_columns": wl.n_seed,
           "outlier_values": f"{wl.mode} U({wl.lo},{wl.hi})" if wl.mode != "scale" else f"x{wl.lo}",
           "sigma_w": wl.sigma_w, "seed": wl.seed, "parallelism": f"replicas x{world}"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        metric = "int8-decomposed matmul TOPS"
        # each step is one bounded sample of the workload (about 12 s with the
        # warm-up samples included, so that the run ends within a few minutes)
        per = max(3.0, min(12.0, 150.0 / max(1, args.steps + args.warmup)))
        for _ in range(args.warmup):
            time_oracle_sample(wl, target_s=per)
        vals, secs, cores, sample = [], 0.0, 0, ""
        for _ in range(args.steps):
            v, dt, cores, sample = time_oracle_sample(wl, target_s=per)
            vals.append(v)
            secs += dt
        value = statistics.median(vals)
        line = {"impl": "reference", "metric": metric, "value": value, "unit": "TOPS", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / max(1, args.steps),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "s8",
                "data": "synthetic", "config": cfg,
                "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample},
                "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    if not torch.cuda.is_available():
        print(json.dumps({"metric": "int8-decomposed matmul TOPS", "error": "no CUDA device"}))
        return 1
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    # all timed work runs on one non-default stream (CUDA graphs cannot be
    # captured on the legacy default stream)
    bench_stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(bench_stream)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
        _pg = torch.distributed.group.WORLD

    from int8_quantized_matmul_02_b200 import build

    build.build()
    pk, pk_kind = peaks()

    cap = min(args.max_outliers, wl.K)
    if args.only:
        # one object alone, for a profiler run: no headline, no CPU baseline
        if args.only == "decode":
            d = run_decode(args.decode_steps, args.warmup, dev, min(args.max_outliers, 4096))
            out = {"us_per_step": d["plain_us"], "us_alone": d["kern_us"], "graph_us": d["graph_us"]}
        elif args.only == "decode_int4":
            out = {f"G{G}": run_int4_decode(args.decode_steps, args.warmup, dev, G) for G in synth.INT4_GROUPS}
            for v in out.values():
                v.pop("wl", None)
        elif args.only == "block_codec":
            out = run_codec(args.steps, args.warmup, dev)
        else:
            out = {}
            for G in synth.GROUP_SIZES:
                rg = run_grouped(wl, G, args.steps, args.warmup, dev, cap)
                out[f"G{G}"] = {"ms_per_step": rg["total_ms"] / args.steps, "n_o": rg["n_o"]}
        print(json.dumps({"only": args.only, "result": out}, default=str), flush=True)
        return 0
    small = wl.M <= 16
    if small:
        r = run_decode(args.steps * 100, args.warmup, dev, cap)
        per_step_s = r["plain_us"] * 1e-6
        value_local = r["bytes"] / per_step_s / 1e9
        metric = "int8-decomposed matmul HBM GB/s (decode M)"
        unit = "GB/s"
        n_o = r["n_o"]
        kern_s = per_step_s
        roof = {"bound": "hbm", "achieved": r["bytes"] / per_step_s / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "basis": "back-to-back step", "alone_us_per_launch": r["kern_us"]}
        launches = 1
    else:
        r = run_gemm_workload(wl, args.steps, args.warmup, dev, rank, cap)
        per_step_s = r["total_ms"] * 1e-3 / args.steps
        value_local = wl.ops / per_step_s / 1e12
        metric = "int8-decomposed matmul TOPS"
        unit = "TOPS"
        n_o = r["n_o"]
        kern_s = statistics.mean(r["kern_ms"]) * 1e-3
        timed_s = r["total_ms"] * 1e-3
        sustained = timed_s >= 2.0
        bf16 = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": wl.ops / kern_s / 1e12, "peak": bf16 * INT8_PER_BF16,
                "unit": "TFLOP/s",
                "peak_note": (f"dense int8 = {INT8_PER_BF16:g} x {pk_kind} bf16 "
                              f"({'sustained' if sustained else 'burst'}) cuBLAS peak"),
                "frac_of_nominal_int8": (wl.ops / kern_s / 1e12) / NOMINAL_INT8_TOPS}
        launches = 4

    per_step_max, value = combine_ranks(per_step_s, value_local * per_step_s, dev, _pg is not None)
    roof["frac"] = roof["achieved"] / roof["peak"]
    kern = "k_decode_int8_sm100" if small else ("k_gemm_int8_2sm" if wl.M > 128 else "k_gemm_int8_sm100")
    roof["traffic"] = recorded_traffic(kern, args.workload)
    roof["kernel"] = kern
    roof["ms_per_launch"] = kern_s * 1e3
    roof["peak_source"] = pk_kind

    cfg["outlier_columns_detected"] = n_o
    cfg["eight_bit_share"] = 1.0 - n_o / wl.K
    cfg["max_outliers"] = cap
    cfg["l2"] = ("inputs larger than L2: X %.0f MB + Wq %.0f MB per step" % (wl.M * wl.K * 2 / 1e6, wl.N * wl.K / 1e6)
                 if not small else "8 rotating prepared weights (8 x %.0f MB > 126 MB L2)" % (wl.N * wl.K / 1e6))

    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_step_max * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "s8", "data": "synthetic", "config": cfg, "roofline": roof,
            "gpu_launches": launches * (args.steps if not small else args.steps * 100)}
    if not small:
        line["clocks"] = r["clocks"]
        e2e_ms, bi, bo = run_e2e(wl, r, max(3, args.steps // 4), dev)
        line["e2e"] = {"value": wl.ops / (e2e_ms * 1e-3) / 1e12 * world, "unit": unit, "h2d_bytes_per_step": bi,
                       "d2h_bytes_per_step": bo, "ms_per_step": e2e_ms}
        for k in ("w", "ws", "X", "Xd", "Y"):
            r.pop(k, None)
        torch.cuda.empty_cache()
        d = None
        if not args.no_decode:
            try:
                d = run_decode(args.decode_steps, args.warmup, dev, min(args.max_outliers, 4096))
            except Exception as exc:  # keep the headline line; say what failed
                line["decode"] = {"error": f"{type(exc).__name__}: {exc}"}
        if d is not None:
            dw = d["wl"]
            step_gbs = d["bytes"] / (d["plain_us"] * 1e-6) / 1e9
            alone_gbs = d["bytes"] / (d["kern_us"] * 1e-6) / 1e9
            line["decode"] = {
                "workload": WORKLOAD_NAMES["decode"], "metric": "HBM GB/s", "unit": "GB/s",
                "value": step_gbs, "us_per_step": d["plain_us"], "graph_us_per_step": d["graph_us"],
                "graph_value": d["bytes"] / (d["graph_us"] * 1e-6) / 1e9,
                "algorithmic_bytes": d["bytes"], "outlier_columns_detected": d["n_o"],
                # the roofline fraction is the step's: forwards back to back, each
                # launched while the previous one finishes (as in a model's
                # layer sequence); the launch alone is reported beside it
                "roofline": {"bound": "hbm", "kernel": "k_decode_int8_sm100", "basis": "back-to-back step",
                             "achieved": step_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": step_gbs / pk["hbm_gbs"], "us_per_launch": d["plain_us"],
                             "peak_source": pk_kind, "traffic": recorded_traffic("k_decode_int8_sm100", "decode")},
                "alone": {"us_per_launch": d["kern_us"], "achieved": alone_gbs, "frac": alone_gbs / pk["hbm_gbs"],
                          "note": "CUDA events around every launch (no overlap with the previous call)"},
                "l2": "8 rotating prepared weights (8 x %.0f MB > 126 MB L2)" % (dw.N * dw.K / 1e6),
            }
            line["gpu_launches"] += args.decode_steps * 2 + max(1, args.decode_steps // 32) * 32
        if not args.no_variants:
            line["decode_int4"] = {}
            for G in synth.INT4_GROUPS:
                try:
                    q = run_int4_decode(args.decode_steps, args.warmup, dev, G)
                except Exception as exc:
                    line["decode_int4"][f"G{G}"] = {"error": f"{type(exc).__name__}: {exc}"}
                    continue
                step_gbs = q["bytes"] / (q["step_us"] * 1e-6) / 1e9
                line["decode_int4"][f"G{G}"] = {
                    "workload": "4-bit weight-only product, decode-shaped FFN up-proj 8x4096x11008, groups of %d" % G,
                    "metric": "HBM GB/s", "unit": "GB/s", "value": step_gbs, "us_per_step": q["step_us"],
                    "algorithmic_bytes": q["bytes"],
                    "roofline": {"bound": "hbm", "kernel": "k_int4_decode_sm100", "basis": "back-to-back step",
                                 "achieved": step_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                 "frac": step_gbs / pk["hbm_gbs"], "peak_source": pk_kind},
                    "alone": {"us_per_launch": q["alone_us"],
                              "frac": q["bytes"] / (q["alone_us"] * 1e-6) / 1e9 / pk["hbm_gbs"]},
                    "l2": "8 rotating prepared weights (8 x %.1f MB > 126 MB L2)" % (q["bytes"] / 1e6),
                }
                line["gpu_launches"] += args.decode_steps + min(args.decode_steps, 400)
            try:
                c = run_codec(args.steps, args.warmup, dev)
                qg = c["quant_bytes"] / c["quant_s"] / 1e9
                dg = c["dequant_bytes"] / c["dequant_s"] / 1e9
                line["block_codec"] = {
                    "workload": "block-wise 8-bit codec, %d fp32 values (one 175B-scale FFN weight's state), "
                                "blocks of %d" % (c["n"], c["B"]),
                    "metric": "HBM GB/s", "unit": "GB/s",
                    "quantise": {"value": qg, "ms": c["quant_s"] * 1e3, "bytes": c["quant_bytes"],
                                 "frac": qg / pk["hbm_gbs"], "kernel": "k_block_quant"},
                    "dequantise": {"value": dg, "ms": c["dequant_s"] * 1e3, "bytes": c["dequant_bytes"],
                                   "frac": dg / pk["hbm_gbs"], "kernel": "k_block_dequant"},
                    "peak": pk["hbm_gbs"], "peak_source": pk_kind, "l2": "input 201 MB > 126 MB L2",
                }
                line["gpu_launches"] += 2 * args.steps
            except Exception as exc:
                line["block_codec"] = {"error": f"{type(exc).__name__}: {exc}"}
        if not args.no_variants:
            line["grouped"] = {}
            for G in synth.GROUP_SIZES:
                try:
                    rg = run_grouped(wl, G, args.steps, args.warmup, dev, cap)
                except Exception as exc:
                    line["grouped"][f"G{G}"] = {"error": f"{type(exc).__name__}: {exc}"}
                    continue
                step_s = rg["total_ms"] * 1e-3 / args.steps
                k_s = statistics.mean(rg["kern_ms"]) * 1e-3
                sus = rg["total_ms"] * 1e-3 >= 2.0
                pk8 = (pk["bf16_tflops_sustained"] if sus else pk["bf16_tflops"]) * INT8_PER_BF16
                line["grouped"][f"G{G}"] = {
                    "workload": "group-wise variant, %s, groups of %d" % (WORKLOAD_NAMES[args.workload], G),
                    "metric": "int8-decomposed matmul TOPS", "unit": "TOPS", "value": wl.ops / step_s / 1e12,
                    "ms_per_step": step_s * 1e3, "frac_of_nominal_int8": wl.ops / step_s / 1e12 / NOMINAL_INT8_TOPS,
                    "outlier_columns_detected": rg["n_o"],
                    "roofline": {"bound": "tensor", "kernel": "k_gemm_int8_grouped", "achieved": wl.ops / k_s / 1e12,
                                 "peak": pk8, "unit": "TFLOP/s", "frac": wl.ops / k_s / 1e12 / pk8,
                                 "ms_per_launch": k_s * 1e3,
                                 "peak_note": "dense int8 = 2 x %s bf16 (%s) cuBLAS peak"
                                              % (pk_kind, "sustained" if sus else "burst")},
                    "clocks": rg["clocks"],
                }
                line["gpu_launches"] += 4 * args.steps
                torch.cuda.empty_cache()
        if not args.no_configs:
            line["configs"] = {}
            for name in ("prefill", "qkv_o0", "qkv_o12", "qkv_o48", "qkv_o123", "qkv_inf"):
                cw = synth.WORKLOADS[name]
                try:
                    rc = run_gemm_workload(cw, args.steps, args.warmup, dev, rank, min(args.max_outliers, cw.K))
                except Exception as exc:
                    line["configs"][name] = {"error": f"{type(exc).__name__}: {exc}"}
                    continue
                step_s = rc["total_ms"] * 1e-3 / args.steps
                k_s = statistics.mean(rc["kern_ms"]) * 1e-3
                sus = rc["total_ms"] * 1e-3 >= 2.0
                pk8 = (pk["bf16_tflops_sustained"] if sus else pk["bf16_tflops"]) * INT8_PER_BF16
                gemm = "k_gemm_int8_2sm" if cw.M > 128 else "k_gemm_int8_sm100"
                line["configs"][name] = {
                    "workload": WORKLOAD_NAMES[name], "metric": "int8-decomposed matmul TOPS", "unit": "TOPS",
                    "value": cw.ops / step_s / 1e12, "ms_per_step": step_s * 1e3,
                    "frac_of_nominal_int8": cw.ops / step_s / 1e12 / NOMINAL_INT8_TOPS,
                    "outlier_columns_detected": rc["n_o"], "eight_bit_share": 1.0 - rc["n_o"] / cw.K,
                    "roofline": {"bound": "tensor", "kernel": gemm, "achieved": cw.ops / k_s / 1e12, "peak": pk8,
                                 "unit": "TFLOP/s", "frac": cw.ops / k_s / 1e12 / pk8, "ms_per_launch": k_s * 1e3,
                                 "peak_note": "dense int8 = 2 x %s bf16 (%s) cuBLAS peak"
                                              % (pk_kind, "sustained" if sus else "burst")},
                    "clocks": rc["clocks"],
                }
                line["gpu_launches"] += 4 * args.steps
                del rc
                torch.cuda.empty_cache()
    else:
        line["e2e"] = None

    if rank == 0 and not args.no_cpu_baseline:
        tops, dt, cores, sample = time_oracle_sample(wl, target_s=12.0)
        if small:
            bytes_per_tops = algorithmic_bytes_decode(wl, n_o) / wl.ops
            line["cpu_baseline"] = {"value": tops * 1e12 * bytes_per_tops / 1e9, "unit": "GB/s", "cores": cores,
                                    "kind": "oracle", "sample": sample, "seconds": dt}
        else:
            line["cpu_baseline"] = {"value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle",
                                    "sample": sample, "seconds": dt}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if _pg is not None:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
