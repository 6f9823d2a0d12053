"""Benchmark of the LLM.int8() matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 175b]

Prints ONE JSON line.  The headline workload is the 175B-scale FFN matmul
(X 4096 x 12288, W 12288 x 49152, 24 seeded outlier columns, threshold 6.0):
throughput in int8 TOPS (2*M*N*K per forward, all K counted) with the
dominant kernel's roofline against the dense-int8 tensor peak.  A "decode"
object adds the decode-shaped FFN up-projection (X 8 x 4096, W 4096 x 11008)
in HBM GB/s against the measured copy bandwidth.

One step = one whole forward (outlier detection, X quantisation, outlier weight
gather, int8 GEMM with fused dequantising epilogue and fp16 outlier product);
the weight is prepared once, outside the timed region.  Inputs are synthetic
and seeded (see int8_quantized_matmul_02_b200.synth).

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
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sms, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, smax = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            sms.append(sm)
            mx = smax
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [s for s in sms if s > 0.5 * max(sms)] or sms
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sms)}


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
        t0.record(stream)
        for i in range(steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    total_ms = t0.elapsed_time(t1)
    kern_ms = [a.elapsed_time(b) for a, b in evs]
    st, n_o = i8.device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")
    return {"total_ms": total_ms, "kern_ms": kern_ms, "n_o": n_o, "clocks": clk.summary(), "w": w, "ws": ws,
            "X": X, "Xd": Xd, "Y": Y}


def run_e2e(wl, state, steps: int, dev):
    """Same metric through the public API with host buffers: pinned X in,
    fp16 Y out, both copies inside the timed region."""
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

def time_oracle_sample(wl, target_s: float = 12.0, max_s: float = 30.0):
    """The CPU oracle, as it stands, on a bounded sample of the workload:
    outlier detection and quantisation of the whole X, then the int8 product,
    outlier product and epilogue for a column slice of W (the weight
    conversion is one-time and excluded).  Returns (TOPS, seconds, cores, sample)."""
    import oracle

    cores = oracle.default_threads()
    X, W, cols = synth.make_inputs(wl)
    Xn = X.numpy()
    # calibrate the column slice with a small probe
    n_probe = 16
    Wp = W[:, :n_probe].contiguous().numpy()
    prep = oracle.prepare_weight(Wp, cols)
    t = time.perf_counter()
    steps = oracle.forward_steps_abc(Xn, prep, wl.threshold)
    t_x = time.perf_counter() - t
    t = time.perf_counter()
    acc = oracle.int8_gemm(steps["xq"], prep["wq"], threads=cores)
    t_probe = time.perf_counter() - t
    per_col = t_probe / n_probe
    n_cols = int(max(16, min(wl.N, (target_s - t_x) / max(per_col, 1e-9))))
    n_cols = n_cols // 16 * 16
    Ws = W[:, :n_cols].contiguous().numpy()
    prep = oracle.prepare_weight(Ws, cols)
    t = time.perf_counter()
    steps = oracle.forward_steps_abc(Xn, prep, wl.threshold)
    acc = oracle.int8_gemm(steps["xq"], prep["wq"], threads=cores)
    o = oracle.outlier_gemm(steps["xo"], steps["wo"])
    oracle.epilogue(acc, steps["ra"], prep["ca"], o)
    dt = time.perf_counter() - t
    ops = 2.0 * wl.M * n_cols * wl.K
    sample = (f"all {wl.M} rows of X through outlier detection and quantisation, then the int8 product, fp16 "
              f"outlier product and epilogue for the first {n_cols} of {wl.N} output columns "
              f"({ops:.3g} int8 ops); weight conversion excluded")
    return ops / dt / 1e12, dt, cores, sample, n_cols


# ----------------------------------------------------------------------------- main

def main():
    global _pg
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="175b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--max-outliers", type=int, default=1024)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=2000)
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
        tops, dt, cores, sample, _ = time_oracle_sample(wl, target_s=min(12.0, 60.0 / max(1, args.steps + args.warmup)))
        vals = []
        for _ in range(args.steps):
            v, dts, _, _, _ = time_oracle_sample(wl, target_s=min(12.0, 60.0 / max(1, args.steps + args.warmup)))
            vals.append(v)
        value = statistics.median(vals) if vals else tops
        line = {"impl": "reference", "metric": metric, "value": value, "unit": "TOPS", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic", "config": cfg,
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
    small = wl.M <= 16
    if small:
        r = run_decode(args.steps * 100, args.warmup, dev, cap)
        per_step_s = r["plain_us"] * 1e-6
        value_local = r["bytes"] / per_step_s / 1e9
        metric = "int8-decomposed matmul HBM GB/s (decode M)"
        unit = "GB/s"
        n_o = r["n_o"]
        kern_s = r["kern_us"] * 1e-6
        roof = {"bound": "hbm", "achieved": r["bytes"] / kern_s / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
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
        d = None
        if not args.no_decode:
            try:
                d = run_decode(args.decode_steps, args.warmup, dev, min(args.max_outliers, 4096))
            except Exception as exc:  # keep the headline line; say what failed
                line["decode"] = {"error": f"{type(exc).__name__}: {exc}"}
        if d is not None:
            dw = d["wl"]
            line["decode"] = {
                "workload": WORKLOAD_NAMES["decode"], "metric": "HBM GB/s", "unit": "GB/s",
                "value": d["bytes"] / (d["plain_us"] * 1e-6) / 1e9,
                "us_per_step": d["plain_us"], "graph_us_per_step": d["graph_us"],
                "graph_value": d["bytes"] / (d["graph_us"] * 1e-6) / 1e9,
                "algorithmic_bytes": d["bytes"], "outlier_columns_detected": d["n_o"],
                "roofline": {"bound": "hbm", "kernel": "k_decode_int8_sm100",
                             "achieved": d["bytes"] / (d["kern_us"] * 1e-6) / 1e9, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": d["bytes"] / (d["kern_us"] * 1e-6) / 1e9 / pk["hbm_gbs"],
                             "us_per_launch": d["kern_us"], "peak_source": pk_kind,
                             "traffic": recorded_traffic("k_decode_int8_sm100", "decode")},
                "l2": "8 rotating prepared weights (8 x %.0f MB > 126 MB L2)" % (dw.N * dw.K / 1e6),
            }
            line["gpu_launches"] += args.decode_steps * 3 + (args.decode_steps // 32) * 32
    else:
        line["e2e"] = None

    if rank == 0 and not args.no_cpu_baseline:
        tops, dt, cores, sample, _ = time_oracle_sample(wl, target_s=12.0)
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
