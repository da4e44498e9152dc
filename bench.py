"""Benchmark of the B200 W4A16 GPTQ linear (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_up] [--no-sweep]

A step is one call of gptq_w4a16_gemm (validate, dispatch, kernel) on the
headline workload: the decode GEMV of the FFN up-projection shape, M=1,
K=5120, N=17408, group 128 (46.0 MB of algorithmic traffic per call).  The
metric is achieved GB/s of algorithmic bytes (packed weights + scales + X + Y,
each moved once).  Inputs are resident in HBM; consecutive steps rotate over
enough distinct copies of the weights that every step reads from HBM, not L2.

With N > 1 (torchrun), every rank runs an independent replica on its own GPU
(the layer needs no exchange between GPUs): value = all ranks' bytes / the
slowest rank's time.  `--impl reference` times the CPU oracle instead (rank 0
only) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int4_weight_only_gptq_b200 import workloads as W  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_up", choices=sorted(WORKLOADS))
    ap.add_argument("--no-sweep", action="store_true")
    return ap.parse_args()


# name -> (problem, description, roofline).  The default is the headline.
WORKLOADS = {
    "decode_up": (lambda: W.decode_up(),
                  "decode GEMV, FFN up-projection: M=1, K=5120, N=17408, group=128", "hbm"),
    "decode_down_m1": (lambda: W.decode_down(1),
                       "decode, FFN down-projection: M=1, K=17408, N=5120, group=32, outliers", "hbm"),
    "decode_down_m16": (lambda: W.decode_down(16),
                        "decode, FFN down-projection: M=16, K=17408, N=5120, group=32, outliers", "hbm"),
    "prefill_m2048": (lambda: W.prefill(2048),
                      "prefill GEMM: M=2048, K=5120, N=17408, group=128", "tensor"),
    "prefill_m8192": (lambda: W.prefill(8192),
                      "prefill GEMM: M=8192, K=5120, N=17408, group=128", "tensor"),
}


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(bytes_per_step: int, steps: int, elapsed_ms_max: float, world: int):
    """(ms per step, whole-job GB/s, per-GPU GB/s) for weak scaling: every
    rank moved bytes_per_step per step; the slowest rank's time counts."""
    ms = elapsed_ms_max / steps
    per_gpu = bytes_per_step / (ms * 1e-3) / 1e9
    return ms, per_gpu * world, per_gpu


def peaks():
    """(HBM GB/s, dense 16-bit TFLOP/s burst, same sustained, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        burst = float(d["bf16_tflops"])
        return (float(d["hbm_gbs"]), burst, float(d.get("bf16_tflops_sustained", burst)),
                "measured")
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def tensor_peak(burst, sustained, src, elapsed_ms, reasons):
    """The burst figure for a kernel timed alone; the sustained one for a
    kernel timed inside a long loop (half a second or more of back-to-back
    launches) or while the power cap was active."""
    long_run = elapsed_ms >= 500.0 or "sw_power_cap" in (reasons or [])
    if long_run:
        return sustained, (f"{src} sustained bf16 figure (timed region {elapsed_ms:.0f} ms"
                           f"{', power cap active' if 'sw_power_cap' in (reasons or []) else ''});"
                           " FP16 dense has the same nominal rate")
    return burst, f"{src} burst bf16 figure (timed region {elapsed_ms:.0f} ms); FP16 dense has the same nominal rate"


def _code_only(text: str) -> str:
    """C/C++ source without its comments, blank space collapsed (string and
    character literals kept whole)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_digest() -> str:
    """Hash of the code of the CUDA sources (comments and blank space do not
    count): ncu counters stay attached to the kernels across edits of their
    comments and are dropped by any change of code."""
    import hashlib
    src = os.path.join(ROOT, "int4_weight_only_gptq_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(src)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(src, name), encoding="utf-8") as f:
                h.update(name.encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_record(kernel_file: str, key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel code (matching digest); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    digest = kernel_source_digest()
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 3 and parts[0] == key and parts[1] == digest:
                    return float(parts[2])
    except OSError:
        pass
    return None


# ---- clocks --------------------------------------------------------------

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index: int, uuid: str | None = None, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        self._stop = threading.Event()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            if uuid:
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByUUID(
                        uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
                except Exception:
                    self.h = None
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---- GPU arm -------------------------------------------------------------

def to_device(p, torch, copies: int):
    x = torch.from_numpy(p.x.view(np.int16)).view(torch.float16).cuda()
    qw0 = torch.from_numpy(p.qweight).cuda()
    s0 = torch.from_numpy(p.scales.view(np.int16)).view(torch.float16).cuda()
    sets = []
    for i in range(copies):
        qw = qw0 if i == 0 else qw0.clone()
        s = s0 if i == 0 else s0.clone()
        xi = x if i == 0 else x.clone()
        y = torch.empty((p.M, p.N), dtype=torch.float16, device="cuda")
        sets.append((xi, qw, s, y))
    return sets


def copies_for(p, l2_bytes: int) -> int:
    per = p.K * p.N // 2 + p.scales.size * 2 + p.M * p.K * 2 + p.M * p.N * 2
    return max(1, math.ceil(2 * l2_bytes / per) + 1)


def hold_device(torch, us: float = 50.0):
    """A short device-side wait enqueued before the start event, outside the
    timed region: the graph replay behind it is already submitted when the
    start event is reached, so the timed region holds the device's work and
    not the host's submission latency (the end-to-end line keeps that)."""
    torch.cuda._sleep(int(us * 2000))


def time_loop(torch, fn, make_argv, steps, warmup, graph=True):
    """Device time per call (ms) of `steps` back-to-back calls fn(*argv[i % n]),
    argv = make_argv(stream handle), after `warmup` untimed calls.

    graph=True: the `steps` calls are captured once in a CUDA graph (each call
    still validates, dispatches and launches through the C ABI while it is
    captured) and the graph is replayed once untimed and once timed, so the
    device runs the calls back to back without waiting for the host.  Else an
    eager loop of calls.  Returns (ms per call, host us per call of the eager
    enqueue loop or None)."""
    stream = torch.cuda.current_stream()
    argv = make_argv(ctypes.c_void_p(stream.cuda_stream))
    n = len(argv)
    for i in range(warmup):
        st = fn(*argv[i % n])
        if st:
            raise RuntimeError(f"status {st}")
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph:
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        with torch.cuda.graph(g, stream=cap):
            av = make_argv(ctypes.c_void_p(cap.cuda_stream))
            for i in range(steps):
                st = fn(*av[i % n])
                if st:
                    raise RuntimeError(f"status {st} while capturing")
        g.replay()
        torch.cuda.synchronize()
        hold_device(torch)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        del g
        return ms, None
    e0.record(stream)
    t0 = time.perf_counter()
    for i in range(steps):
        fn(*argv[i % n])
    host_us = (time.perf_counter() - t0) * 1e6 / steps
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, host_us


def gemm_argv(p, sets, kernel=0):
    def make(sh):
        out = []
        for (x, qw, s, y) in sets:
            a = (ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(qw.data_ptr()),
                 ctypes.c_void_p(s.data_ptr()), p.M, p.K, p.N, p.group,
                 ctypes.c_void_p(y.data_ptr()), sh)
            out.append(a if kernel == 0 else a + (kernel,))
        return out
    return make


def time_gemm(lib, torch, p, steps, warmup, kernel=0, l2_bytes=0, graph=True):
    """Device time per call (ms) of back-to-back calls through the C ABI,
    rotating enough copies of the inputs that each call reads from HBM."""
    copies = copies_for(p, l2_bytes) if l2_bytes else 1
    sets = to_device(p, torch, copies)
    fn = lib.gptq_w4a16_gemm if kernel == 0 else lib.gptq_w4a16_gemm_kernel
    ms, _ = time_loop(torch, fn, gemm_argv(p, sets, kernel), steps, warmup, graph)
    return ms, copies


def time_grouped(lib, torch, ps, steps, warmup, l2_bytes):
    """Device time per call (ms) of back-to-back grouped calls (linears sharing
    X), rotating enough weight copies that they do not stay in L2."""
    total = sum(p.algorithmic_bytes for p in ps)
    copies = max(1, -(-2 * l2_bytes // total) + 1)
    keep, per_copy = [], []
    M, K, count = ps[0].M, ps[0].K, len(ps)
    x = torch.from_numpy(ps[0].x.view(np.int16)).view(torch.float16).cuda()
    for c in range(copies):
        qws = [torch.from_numpy(p.qweight).cuda() for p in ps]
        ss = [torch.from_numpy(p.scales.view(np.int16)).view(torch.float16).cuda() for p in ps]
        ys = [torch.empty((M, p.N), dtype=torch.float16, device="cuda") for p in ps]
        keep += qws + ss + ys
        qa = (ctypes.c_void_p * count)(*[ctypes.c_void_p(t.data_ptr()) for t in qws])
        sa = (ctypes.c_void_p * count)(*[ctypes.c_void_p(t.data_ptr()) for t in ss])
        na = (ctypes.c_int64 * count)(*[p.N for p in ps])
        ya = (ctypes.c_void_p * count)(*[ctypes.c_void_p(t.data_ptr()) for t in ys])
        per_copy.append((qa, sa, na, ya))

    def make(sh):
        return [(ctypes.c_void_p(x.data_ptr()), qa, sa, na, count, M, K, ps[0].group, ya, sh)
                for (qa, sa, na, ya) in per_copy]
    ms, _ = time_loop(torch, lib.gptq_w4a16_gemm_grouped, make, steps, warmup)
    return ms


def time_asym(lib, torch, p, qzeros, steps, warmup, l2_bytes):
    """Device time per call (ms) of back-to-back gptq_w4a16_gemm_asym calls,
    rotating weight copies past the L2 like time_gemm."""
    copies = copies_for(p, l2_bytes) if l2_bytes else 1
    sets = to_device(p, torch, copies)
    zs = [torch.from_numpy(qzeros).cuda() for _ in range(copies)]
    v = ctypes.c_void_p

    def make(sh):
        return [(v(x.data_ptr()), v(qw.data_ptr()), v(s.data_ptr()), v(z.data_ptr()), p.M, p.K,
                 p.N, p.group, v(y.data_ptr()), sh) for (x, qw, s, y), z in zip(sets, zs)]
    ms, _ = time_loop(torch, lib.gptq_w4a16_gemm_asym, make, steps, warmup)
    return ms


def time_gidx(lib, torch, p, g_idx, steps, warmup, l2_bytes):
    """Device time per call (ms) of back-to-back gptq_w4a16_gemm_gidx calls
    (act-order weights), rotating weight copies past the L2 like time_gemm."""
    copies = copies_for(p, l2_bytes) if l2_bytes else 1
    sets = to_device(p, torch, copies)
    gi = torch.from_numpy(g_idx).cuda()
    v = ctypes.c_void_p
    ng = p.scales.shape[0]

    def make(sh):
        return [(v(x.data_ptr()), v(qw.data_ptr()), v(s.data_ptr()), v(gi.data_ptr()), p.M, p.K,
                 p.N, ng, v(y.data_ptr()), sh) for (x, qw, s, y) in sets]
    ms, _ = time_loop(torch, lib.gptq_w4a16_gemm_gidx, make, steps, warmup)
    return ms


def time_lora(lib, torch, p, ad, steps, warmup, l2_bytes):
    """Device time per call (ms) of back-to-back gptq_w4a16_gemm_lora calls
    (the adapter's down-projection launch and the layer launch), rotating
    weight copies past the L2 like time_gemm."""
    copies = copies_for(p, l2_bytes) if l2_bytes else 1
    sets = to_device(p, torch, copies)
    a = torch.from_numpy(ad.lora_a.view(np.int16)).view(torch.float16).cuda()
    b = torch.from_numpy(ad.lora_b.view(np.int16)).view(torch.float16).cuda()
    t = torch.empty((p.M, ad.rank), dtype=torch.float16, device="cuda")
    v = ctypes.c_void_p

    def make(sh):
        return [(v(x.data_ptr()), v(qw.data_ptr()), v(s.data_ptr()), p.M, p.K, p.N, p.group,
                 v(a.data_ptr()), v(b.data_ptr()), ad.rank, v(t.data_ptr()), v(y.data_ptr()), sh)
                for (x, qw, s, y) in sets]
    ms, _ = time_loop(torch, lib.gptq_w4a16_gemm_lora, make, steps, warmup)
    return ms


def hbm_entry(p, ms, hbm, extra_bytes=0):
    gbs = (p.algorithmic_bytes + extra_bytes) / (ms * 1e-3) / 1e9
    return {"M": p.M, "K": p.K, "N": p.N, "group": p.group, "ms": round(ms, 5),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(gbs / hbm, 3)}}


def tensor_entry(p, ms, peak, extra_flops=0):
    tfl = (p.flops + extra_flops) / (ms * 1e-3) / 1e12
    return {"M": p.M, "K": p.K, "N": p.N, "group": p.group, "ms": round(ms, 4),
            "roofline": {"bound": "tensor", "achieved": round(tfl, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tfl / peak, 3)}}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from int4_weight_only_gptq_b200 import binding

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    lib = binding.load()
    props = torch.cuda.get_device_properties(local_rank)
    l2 = props.L2_cache_size
    make, desc, bound = WORKLOADS[args.workload]
    p = make()
    bytes_per_step = p.algorithmic_bytes
    # HBM-bound workloads rotate over copies whose total exceeds twice the L2;
    # the tensor-bound ones move more than the L2 per call anyway
    copies = copies_for(p, l2) if bound == "hbm" else 1
    sets = to_device(p, torch, copies)
    fn = lib.gptq_w4a16_gemm
    make_argv = gemm_argv(p, sets)
    stream = torch.cuda.current_stream()
    argv = make_argv(ctypes.c_void_p(stream.cuda_stream))
    warm = max(3, args.warmup)
    for i in range(warm):
        st = fn(*argv[i % copies])
        if st:
            raise RuntimeError(f"gptq_w4a16_gemm returned {st}: {binding.status_string(st)}")
    torch.cuda.synchronize()
    # the timed steps, captured once as a CUDA graph of `steps` library calls
    # (each call validates, dispatches and launches while it is captured)
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    with torch.cuda.graph(graph, stream=cap):
        av = make_argv(ctypes.c_void_p(cap.cuda_stream))
        for i in range(args.steps):
            st = fn(*av[i % copies])
            if st:
                raise RuntimeError(f"gptq_w4a16_gemm returned {st} while captured")
    graph.replay()  # untimed: the graph's first replay
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank, str(getattr(props, "uuid", "")) or None) as clk:
        hold_device(torch)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = max_over_ranks(e0.elapsed_time(e1), "cuda")
    del graph
    # the same steps as an eager loop of calls (host enqueue between calls)
    eager_ms, host_us = time_loop(torch, fn, make_argv, args.steps, 0, graph=False)
    eager_ms = max_over_ranks(eager_ms, "cuda")
    if binding.device_error() != 0:
        raise RuntimeError("a kernel reported a bounded-wait timeout")
    ms, value, per_gpu = aggregate(bytes_per_step, args.steps, elapsed_ms, world)
    if bound == "tensor":  # the same aggregation in TFLOP/s
        value = value * p.flops / bytes_per_step / 1e3
        per_gpu = per_gpu * p.flops / bytes_per_step / 1e3

    # end to end through the public API with host buffers: pinned X in, Y out
    xh = torch.from_numpy(p.x.view(np.int16)).view(torch.float16).pin_memory()
    yh = torch.empty((p.M, p.N), dtype=torch.float16).pin_memory()
    e2 = []
    for rep in range(2):
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 500 if bound == "hbm" else 20))
        a0.record(stream)
        for i in range(n_e2e):
            xs, qws, ss, ys = sets[i % copies]
            xs.copy_(xh, non_blocking=True)
            binding.gemm(xs, qws, ss, p.group, out=ys, stream=stream)
            yh.copy_(ys, non_blocking=True)
        a1.record(stream)
        torch.cuda.synchronize()
        e2.append(a0.elapsed_time(a1) / n_e2e)
    e2e_ms = max_over_ranks(min(e2), "cuda")

    hbm, tf_burst, tf_sust, src = peaks()
    out = None
    if rank == 0:
        clocks = clk.summary()
        kernel_id, split = binding.select(p.M, p.K, p.N, p.group)
        traffic = traffic_record("decode.cu", f"{args.workload}")
        if bound == "hbm":
            metric = "W4A16 GEMM decode GB/s (algorithmic bytes: packed weights + scales + X + Y)"
            unit, peak, punit = "GB/s", hbm, "GB/s"
            peak_src = ("measured (MEASURED_PEAKS.json hbm_gbs)" if src == "measured"
                        else "fallback 6.65 TB/s")
            e2e_val = bytes_per_step * world / (e2e_ms * 1e-3) / 1e9
            eager_val = bytes_per_step / (eager_ms * 1e-3) / 1e9
        else:
            metric = "W4A16 GEMM prefill TFLOP/s (2*M*K*N)"
            unit, punit = "TFLOP/s", "TFLOP/s"
            peak, peak_src = tensor_peak(tf_burst, tf_sust, src, elapsed_ms,
                                         clocks.get("reasons") if clocks else None)
            e2e_val = p.flops * world / (e2e_ms * 1e-3) / 1e12
            eager_val = p.flops / (eager_ms * 1e-3) / 1e12
        out = {
            "metric": metric,
            "value": round(value, 1), "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": warm, "ms_per_step": round(ms, 6),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp16 x int4 -> fp32 acc -> fp16", "data": "synthetic (seeded, PCG64 seed 0)",
            "config": {"workload": desc, "M": p.M, "K": p.K, "N": p.N, "group": p.group,
                       "bytes_per_step": bytes_per_step,
                       "l2": f"rotating {copies} input copies ({copies * bytes_per_step / 1e6:.0f} MB > 2x L2 {l2 / 1e6:.0f} MB)",
                       "timing": "the steps captured once as a CUDA graph of library calls, replayed once untimed and once timed (CUDA events on the replay stream; a 50 us device-side wait is queued before the start event, so the timed region holds no host submission latency)",
                       "parallelism": f"replicas x{world} (no exchange)",
                       "kernel": {1: "decode", 2: "prefill"}.get(kernel_id, kernel_id),
                       "split_k_ctas": split},
            "roofline": {"bound": bound, "achieved": round(per_gpu, 1), "peak": peak,
                         "unit": punit, "frac": round(per_gpu / peak, 4),
                         "peak_source": peak_src, "traffic": traffic},
            "eager": {"value": round(eager_val, 1), "unit": unit, "ms_per_step": round(eager_ms, 6),
                      "host_us_per_call": round(host_us, 2),
                      "note": "the same steps as a Python loop of C-ABI calls (no graph)"},
            "e2e": {"value": round(e2e_val, 1),
                    "unit": unit, "ms_per_step": round(e2e_ms, 6),
                    "h2d_bytes_per_step": int(p.M * p.K * 2),
                    "d2h_bytes_per_step": int(p.M * p.N * 2),
                    "note": "eager loop: pinned host X -> device, gptq_w4a16_gemm, device Y -> pinned host; weights resident"},
            "gpu_launches": args.steps,
            "clocks": clocks,
        }
    if not args.no_sweep and world == 1:
        sweep = run_sweep(lib, torch, l2, hbm, tf_burst)
        if rank == 0:
            # the long sweep on its own line first; the contract line stays short
            print(json.dumps({"sweep": sweep}), flush=True)
            out.update(headline_keys(sweep))
    if rank == 0:
        cb = cpu_baseline(p, bytes_per_step, bound,
                          y_gpu=yh.view(torch.int16).numpy().view(np.float16))
        parity = cb.pop("parity", None)
        out["cpu_baseline"] = cb
        if parity is not None:
            out["parity"] = parity
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def headline_keys(sweep):
    """The other halves of the metric, compact, for the contract line: prefill
    at M = 2048 and 8192 (tensor roofline), the down-projection decode at
    M = 16 and the mid-M up-projection at M = 64 (HBM roofline)."""
    pick = lambda names: {n.split("_")[-1]: sweep[n] for n in names if n in sweep}
    return {"prefill": pick(["prefill_M2048", "prefill_M8192"]),
            "decode_down": pick(["decode_down_M1", "decode_down_M16"]),
            "midm": pick(["midm_up_M48", "midm_up_M64"])}


def run_sweep(lib, torch, l2, hbm, tf):
    """The other workloads: decode GB/s, prefill TFLOP/s, each with its
    roofline fraction (HBM: measured copy bandwidth; tensor: measured burst)."""
    res = {}

    def hbm_case(name, p, steps=300):
        ms, copies = time_gemm(lib, torch, p, steps, 20, l2_bytes=l2)
        res[name] = hbm_entry(p, ms, hbm)

    def tc_case(name, p, steps=30):
        ms, _ = time_gemm(lib, torch, p, steps, 5)
        res[name] = tensor_entry(p, ms, tf)

    for M in (1, 2, 4, 8, 16, 32):
        hbm_case(f"decode_down_M{M}", W.decode_down(M))
    # between the kernels: decode up to M = 64, pair prefill above
    for M in (24, 32, 48, 64, 96, 128):
        hbm_case(f"midm_up_M{M}", W.make_problem(M, 5120, 17408, 128, seed=0), steps=100)
    for M in (512, 2048, 8192):
        tc_case(f"prefill_M{M}", W.prefill(M))
    for g in W.GROUP_SIZES:
        hbm_case(f"square_g{g}_M1", W.group_sweep(g, 1))
        hbm_case(f"square_g{g}_M16", W.group_sweep(g, 16))
        tc_case(f"square_g{g}_M4096", W.group_sweep(g, 4096))
    for name, K, N, count in W.LAYER_LINEARS:
        for M in (1, 16):
            hbm_case(f"layer_{name}_M{M}", W.layer_linear(name, M))
        tc_case(f"layer_{name}_M4096", W.layer_linear(name, 4096))
    for M in (1, 16, 4096):
        total = sum(res[f"layer_{n}_M{M}"]["ms"] * c for n, _, _, c in W.LAYER_LINEARS)
        res[f"layer_total_M{M}_ms"] = round(total, 4)
    # shared-input linears in one call (q/k/v: 3 x 5120->5120; gate+up: 2 x 5120->17408)
    for name, count, N in (("qkv", 3, 5120), ("gate_up", 2, 17408)):
        for M in (1, 16):
            ps = [W.make_problem(M, 5120, N, 128, seed=i) for i in range(count)]
            ms = time_grouped(lib, torch, ps, 200, 20, l2)
            gbs = sum(p.algorithmic_bytes for p in ps) / (ms * 1e-3) / 1e9
            res[f"grouped_{name}_M{M}"] = {"ms": round(ms, 5), "GB/s": round(gbs, 1),
                                           "frac_hbm": round(gbs / hbm, 3)}
    # LoRA adapter (rank 32) on the up-projection: both launches of one call;
    # the plain layer at the same M is timed beside it
    for M in (1, 16, 2048):
        p = W.make_problem(M, 5120, 17408, 128, seed=0)
        ad = W.make_adapter(5120, 17408, 32, seed=0)
        steps = 200 if M <= 16 else 30
        ms = time_lora(lib, torch, p, ad, steps, 10, l2)
        plain, _ = time_gemm(lib, torch, p, steps, 10, l2_bytes=l2)
        entry = {"ms": round(ms, 5), "plain_ms": round(plain, 5)}
        if M <= 16:
            gbs = (p.algorithmic_bytes + ad.extra_bytes(M)) / (ms * 1e-3) / 1e9
            entry.update({"GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)})
        else:
            tfl = (p.flops + ad.extra_flops(M)) / (ms * 1e-3) / 1e12
            entry.update({"TFLOP/s": round(tfl, 1), "frac_tensor": round(tfl / tf, 3)})
        res[f"lora_r32_up_M{M}"] = entry
    # asymmetric zero points on the up-projection; the symmetric layer beside it
    for M in (1, 16, 2048):
        p = W.make_problem(M, 5120, 17408, 128, seed=0)
        qz = W.make_qzeros(p.scales.shape[0], p.N, seed=0)
        steps = 200 if M <= 16 else 30
        ms = time_asym(lib, torch, p, qz, steps, 10, l2)
        plain, _ = time_gemm(lib, torch, p, steps, 10, l2_bytes=l2)
        entry = {"ms": round(ms, 5), "symmetric_ms": round(plain, 5)}
        if M <= 16:
            gbs = (p.algorithmic_bytes + qz.size * 4) / (ms * 1e-3) / 1e9
            entry.update({"GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)})
        else:
            tfl = p.flops / (ms * 1e-3) / 1e12
            entry.update({"TFLOP/s": round(tfl, 1), "frac_tensor": round(tfl / tf, 3)})
        res[f"asym_up_M{M}"] = entry
    # act order (a group index per input channel, GPTQ's desc_act order) on
    # the up- and down-projections; the plain layer beside it
    for name, mk, Ms in (("up", lambda M: W.make_problem(M, 5120, 17408, 128, seed=0),
                          (1, 16, 64, 2048)),
                         ("down", W.decode_down, (1, 16))):
        for M in Ms:
            p = mk(M)
            g = W.make_gidx(p.K, p.group, seed=0, kind="perm")
            steps = 200 if M <= 64 else 20
            ms = time_gidx(lib, torch, p, g, steps, 10, l2)
            plain, _ = time_gemm(lib, torch, p, steps, 10, l2_bytes=l2)
            entry = {"ms": round(ms, 5), "plain_ms": round(plain, 5)}
            if M <= 64:
                gbs = (p.algorithmic_bytes + g.size * 4) / (ms * 1e-3) / 1e9
                entry.update({"GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)})
            else:
                tfl = p.flops / (ms * 1e-3) / 1e12
                entry.update({"TFLOP/s": round(tfl, 1), "frac_tensor": round(tfl / tf, 3)})
            res[f"gidx_{name}_M{M}"] = entry
    return res


# ---- CPU oracle ----------------------------------------------------------

def parity_on_rows(y_gpu, ref, rows):
    """The required error measure on the sampled rows (every column):
    max |y - y_ref| / (1 + |y_ref|), y the layer's FP16 output, y_ref the
    binary64 oracle."""
    y = np.asarray(y_gpu, dtype=np.float64)[rows]
    ref = np.asarray(ref, dtype=np.float64)
    if y.shape != ref.shape:
        raise ValueError(f"shapes {y.shape} and {ref.shape}")
    err = float(np.max(np.abs(y - ref) / (1.0 + np.abs(ref)))) if y.size else 0.0
    return {"max_rel_err": err, "bound": 1e-2, "within": bool(err <= 1e-2 and np.all(np.isfinite(y))),
            "rows": [int(r) for r in rows], "cols": "all", "against": "binary64 oracle"}


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def cpu_baseline(p, bytes_per_step, bound="hbm", budget_s: float = 8.0, y_gpu=None):
    """The oracle as it stands on a bounded sample of the same workload, in two
    variants: OpenMP over output columns on every host thread (the line's
    value), and one thread.  Every row when M <= 16, else four rows (first,
    last, two inside); the single-thread variant takes a column slice of those
    rows.  Each is repeated for about budget_s and scaled to the metric's unit
    by the share of the work it did.  With y_gpu (the layer's output for the
    same inputs) the oracle's rows also give the parity error."""
    import oracle
    oracle.build()
    threads = oracle.get_threads()
    rows = list(range(p.M)) if p.M <= 16 else sorted({0, p.M // 3, 2 * p.M // 3, p.M - 1})
    n, t0 = 0, time.perf_counter()
    while True:
        ref = oracle.gemm_rows(p.x, p.qweight, p.scales, p.group, rows)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    per = el / n
    share = len(rows) / p.M

    def rate(share_of_work, seconds):
        if bound == "hbm":
            return bytes_per_step * share_of_work / seconds / 1e9, "GB/s"
        return p.flops * share_of_work / seconds / 1e12, "TFLOP/s"

    value, unit = rate(share, per)
    what = "whole call(s) of the workload" if share == 1 else f"calls on {len(rows)} of {p.M} rows"
    out = {"value": round(value, 6), "unit": unit, "cores": threads, "kind": "oracle",
           "sample": f"{n} {what} ({el:.1f} s, {threads} OpenMP threads over output columns)",
           "s_per_call": round(per, 4), "cpu_model": cpu_model(),
           "host_threads": os.cpu_count()}
    # one thread: a slice of the columns of the same rows
    n_cols = min(p.N, 1088)
    cols = np.arange(n_cols, dtype=np.int64)
    ms_ = np.repeat(np.asarray(rows, dtype=np.int64), n_cols)
    ns_ = np.tile(cols, len(rows))
    try:
        oracle.set_threads(1)
        n1, t1 = 0, time.perf_counter()
        while True:
            oracle.gemm_entries(p.x, p.qweight, p.scales, p.group, ms_, ns_)
            n1 += 1
            el1 = time.perf_counter() - t1
            if el1 >= budget_s or n1 >= 1000:
                break
    finally:
        oracle.set_threads(threads)
    share1 = len(rows) * n_cols / (p.M * p.N)
    v1, _ = rate(share1, el1 / n1)
    out["single_thread"] = {"value": round(v1, 6), "unit": unit, "cores": 1,
                            "sample": f"{n1} calls on {len(rows)} row(s) x {n_cols} of {p.N} "
                                      f"columns ({el1:.1f} s, one thread)"}
    if y_gpu is not None:
        try:
            out["parity"] = parity_on_rows(y_gpu, ref, rows)
        except Exception as e:  # the timing stands; the comparison reports why it failed
            out["parity"] = {"error": f"{type(e).__name__}: {e}"}
    return out


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, each step one oracle call
    on a column slice of the workload (every k, every row), so that a step
    takes a fraction of a second; GB/s counts the slice's share of the bytes."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    make, desc, bound = WORKLOADS[args.workload]
    p = make()
    import oracle
    oracle.build()
    threads = oracle.get_threads()
    n_cols = 1088  # N / 16 for the up-projection
    frac = n_cols / p.N
    rows = np.repeat(np.arange(p.M, dtype=np.int64), n_cols)
    warm = min(max(3, args.warmup), 3)
    times = []
    for i in range(warm + args.steps):
        c0 = (i * n_cols) % (p.N - n_cols + 1)
        cols = np.tile(np.arange(c0, c0 + n_cols, dtype=np.int64), p.M)
        t0 = time.perf_counter()
        oracle.gemm_entries(p.x, p.qweight, p.scales, p.group, rows, cols)
        if i >= warm:
            times.append(time.perf_counter() - t0)
        if sum(times) > 90:
            break
    ms = 1e3 * sum(times) / len(times)
    v = frac * p.algorithmic_bytes / (ms * 1e-3) / 1e9
    sample = (f"{len(times)} steps, each all {p.M} row(s) x {n_cols} of {p.N} columns "
              f"(1/16 of the workload), {threads} OpenMP threads over output entries")
    print(json.dumps({
        "impl": "reference", "metric": "W4A16 GEMM decode GB/s (algorithmic bytes: packed weights + scales + X + Y)",
        "value": round(v, 4), "unit": "GB/s", "n_gpus": world, "steps": len(times),
        "warmup": warm, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic (seeded, PCG64 seed 0)",
        "config": {"workload": desc, "M": p.M, "K": p.K, "N": p.N, "group": p.group},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
