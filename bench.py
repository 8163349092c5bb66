#!/usr/bin/env python
"""Benchmark of the DCNv4 core operator on B200: one forward + backward step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload NAME] [--softmax] [--no-linear] [--no-cpu-baseline] [--no-e2e]
    python bench.py --profile [--workload NAME] [--linear] --steps K --warmup W   (for ncu)

A step is one pass of the whole path over one batch: dcn4_forward followed by
dcn4_backward on the first-stage backbone workload (N64 H56 W56 C64 G4, C'=16,
3x3, fp16; inputs seeded, see dcn4_inputs).  Inputs are resident in HBM; the
L2 cache is flushed (a 256 MiB write) between timed steps, outside the timed
events.  Each step is timed with CUDA events on the launching stream, with a
barrier + synchronize around the K timed steps; multi-GPU runs (torchrun, one
rank per GPU, NCCL) report the max over ranks.  Every rank runs the full
batch: the operator is independent per image, so there is no collective on the
data path (weak scaling, replicas).

Rank 0 prints one JSON line.  value = microseconds per forward+backward step
(lower is better); the line also carries per-kernel times, achieved HBM GB/s
against the algorithmic byte model, the roofline of the dominant launch, an
end-to-end figure through host buffers, clocks sampled during the timed loop,
and a CPU-oracle baseline.

--softmax runs the same step with the masks normalised by a softmax over the
K points of each (pixel, group) (the DCNv3 form of the operator).

The "linear" object (skipped with --no-linear) times the layer with its
producer: the forward with the producer fused in (dcn4_forward_linear:
offset_mask = x W^T + b formed per tile on the tensor cores; fp16/bf16
workloads) against the producer as a separate library GEMM (cuBLAS) followed
by dcn4_forward; and the layer's backward dcn4_backward_linear (the
aggregation's backward, then grad_x = g W, grad_W = g^T x, grad_b on the
tensor cores in libdcn4) against dcn4_backward followed by cuBLAS products.
The "projection" object (also skipped with --no-linear) times the output
projection fused behind the operator (dcn4_forward_proj: y = core W^T + b per
tile on the tensor cores, W [C, C]) against dcn4_forward followed by cuBLAS's
linear layer, and dcn4_backward_proj against cuBLAS products followed by
dcn4_backward.

--profile runs warm-up + steps untimed passes of the workload (forward and
backward; with --linear also the fused forward and dcn4_backward_linear) and
prints no JSON line: a fixed launch sequence for ncu captures.

The line also carries "per_config": forward and backward µs per call,
achieved GB/s and fractions of the measured copy bandwidth and of 8 TB/s for
every workload of the configuration table (tiny fp32, first-stage fp16,
third-stage bf16, high-resolution fp16, training-step bf16), each stage timed
over --config-reps calls with the L2 flushed before every call.

--impl reference times the CPU oracle (the only other implementation of the
operator) on the host cores: each step is one forward + backward call on the
whole batch when the run fits about REFERENCE_BUDGET_S seconds, else on a
sample of at least one image per host thread (value scaled to the batch;
ms_per_step is always the measured step).  cpu_baseline in the native line
times the same calls for about --cpu-seconds of CPU work.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import dcn4_inputs as gen  # noqa: E402

METRIC = "DCNv4 core fwd/bwd µs per call and achieved HBM GB/s (% of B200 peak)"
L2_FLUSH_BYTES = 256 << 20
REFERENCE_BUDGET_S = 150.0
FALLBACK_HBM_GBS = 6650.0
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


# ---------------------------------------------------------------------------
# Byte model (compulsory HBM traffic per call)
# ---------------------------------------------------------------------------

def byte_model(w: gen.Workload) -> dict:
    """Compulsory HBM bytes per call.  forward: value + offset_mask read, out
    written.  backward: value + offset_mask + grad_out read, grad_value +
    grad_offset_mask written.  Per backward kernel: the offset/mask stage reads
    value, offset_mask, grad_out and writes grad_offset_mask; the value stage
    reads offset_mask and grad_out and writes grad_value."""
    b = ELEM_BYTES[w.dtype]
    value = w.N * w.H * w.W * w.C * b
    om = w.N * w.Ho * w.Wo * w.P * b
    out = w.N * w.Ho * w.Wo * w.C * b
    return {"fwd": value + om + out, "bwd": value + om + out + value + om,
            "bwd_offset_mask": value + om + out + om, "bwd_value": om + out + value}


KERNELS = {"fwd": "forward_kernel", "bwd_offset_mask": "samples_kernel", "bwd_value": "value_kernel"}


# Sources each kernel is built from: its own translation unit, the shared device
# helpers, the host side that sets its launch geometry, and the ABI header.
KERNEL_SOURCES = {
    "forward_kernel": ["csrc/dcn4_forward.cu"],
    "samples_kernel": ["csrc/dcn4_backward.cu"],
    "value_kernel": ["csrc/dcn4_backward.cu"],
}
COMMON_SOURCES = ["csrc/dcn4_common.cuh", "csrc/dcn4_api.cu", "../include/dcn4.h"]


def kernel_sources_sha(kernel: str) -> str:
    """sha256 over the sources `kernel` is built from: a DRAM-traffic capture is
    only reported while the kernel is the one it measured."""
    import hashlib
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "deformable_convolution_sampling_b200")
    for rel in KERNEL_SOURCES[kernel] + COMMON_SOURCES:
        with open(os.path.normpath(os.path.join(pkg, rel)), "rb") as fh:
            h.update(os.path.basename(rel).encode())
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from profiles/dram_traffic.txt,
    or None when absent or captured from other kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    sha = kernel_sources_sha(kernel)
    for line in lines:
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload:
            return int(float(parts[2])) if parts[3] == sha else None
    return None


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


# ---------------------------------------------------------------------------
# Clock sampling (nvidia-smi in the background during the timed loop)
# ---------------------------------------------------------------------------

CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int, period_ms: int = 100):
        self.samples: list[tuple[float, list[str]]] = []
        self.proc = None
        self.gpu_index = gpu_index
        self.period_ms = period_ms
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_QUERY}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.period_ms), "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()


def summarize_clocks(samples, t0: float, t1: float) -> dict:
    """Median SM clock and the throttle reasons seen in [t0, t1] (all samples if none fall inside)."""
    inside = [s for t, s in samples if t0 <= t <= t1]
    window = "timed loop"
    if not inside:
        inside = [s for _, s in samples]
        window = "whole run (timed loop shorter than the sampling period)"
    if not inside:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": "unavailable"}
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    sm, smax, reasons = [], [], set()
    for s in inside:
        try:
            sm.append(float(s[1]))
            smax.append(float(s[2]))
        except (ValueError, IndexError):
            continue
        for i, n in enumerate(names):
            if len(s) > 5 + i and s[5 + i].lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ---------------------------------------------------------------------------
# Distributed plumbing
# ---------------------------------------------------------------------------

def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline / reference arm)
# ---------------------------------------------------------------------------

def oracle_call_seconds(w: gen.Workload, inp: dict, threads: int) -> float:
    """Wall seconds of one oracle forward + backward on the images of `inp`."""
    import oracle
    prob = oracle.Problem(dtype=w.dtype, location_fp32=True, **{**w.geometry(), "N": inp["value"].shape[0]})
    t0 = time.perf_counter()
    oracle.forward(prob, inp["value"], inp["offset_mask"], nthreads=threads)
    oracle.backward(prob, inp["value"], inp["offset_mask"], inp["grad_out"], nthreads=threads)
    return time.perf_counter() - t0


def oracle_sample(w: gen.Workload, images: int) -> dict:
    sub = gen.custom(**{**w.__dict__, "N": images, "name": w.name + "_sample"})
    return gen.make_inputs(sub, tail_fill=0.0)


def oracle_images(w: gen.Workload, seconds_per_call: float, threads: int) -> tuple[int, float]:
    """Images per oracle call so that one call takes about `seconds_per_call`: the
    whole batch when it fits, else a sample of at least `threads` images (the
    oracle's backward runs one image per thread).  Returns (images, estimated
    seconds of one whole-batch call)."""
    probe_n = max(1, min(w.N, threads))
    per_img = oracle_call_seconds(w, oracle_sample(w, probe_n), threads) / probe_n
    full = per_img * w.N
    if full <= seconds_per_call:
        return w.N, full
    n = int(seconds_per_call // max(per_img, 1e-9))
    return max(probe_n, min(w.N, n)), full


def time_oracle(w: gen.Workload, target_s: float) -> dict:
    """The oracle as a baseline: forward + backward calls on the host cores for
    about target_s seconds of CPU work, in µs per whole-batch call."""
    import oracle
    threads = oracle.host_threads()
    images, _ = oracle_images(w, target_s, threads)
    inp = oracle_sample(w, images)
    secs = []
    while not secs or (sum(secs) < target_s and len(secs) < 20):
        secs.append(oracle_call_seconds(w, inp, threads))
    per_call = statistics.mean(secs)
    us_full = per_call * 1e6 * w.N / images
    used = min(threads, images)
    scaled = "" if images == w.N else f", scaled x{w.N / images:g} to the {w.N}-image batch"
    return {"value": round(us_full, 1), "unit": "us/call", "cores": used, "kind": "oracle",
            "sample": f"{len(secs)} calls of forward+backward on {images} of {w.N} images with {used} threads "
                      f"(of {threads}), {sum(secs):.2f} s of CPU work{scaled}"}


def run_reference(args, w: gen.Workload) -> dict:
    """The oracle as the reference arm: each step is one forward + backward call on
    the host cores, on the whole batch when the --steps/--warmup run fits about
    REFERENCE_BUDGET_S seconds, else on a sample of images (value scaled to the
    batch; ms_per_step is always the measured step)."""
    import oracle
    rank, world, _ = dist_env()
    if rank != 0:
        return {}
    threads = oracle.host_threads()
    images, _ = oracle_images(w, REFERENCE_BUDGET_S / (args.steps + args.warmup), threads)
    inp = oracle_sample(w, images)
    for _ in range(args.warmup):
        oracle_call_seconds(w, inp, threads)
    secs = [oracle_call_seconds(w, inp, threads) for _ in range(args.steps)]
    step_s = statistics.mean(secs)
    us = step_s * 1e6 * w.N / images
    used = min(threads, images)
    sample = (f"each step: forward+backward on {images} of {w.N} images with {used} threads (of {threads}), "
              f"{step_s:.3f} s" + ("" if images == w.N else f"; value scaled x{w.N / images:g} to the batch"))
    return {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "us/call",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": f"{w.name}: {w.describe()}, forward+backward",
                                        "parallelism": "oracle on host cores", "images_per_step": images},
        "cpu_baseline": {"value": round(us, 1), "unit": "us/call", "cores": used, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(us, 1), "unit": "us/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# Native arm
# ---------------------------------------------------------------------------

def run_native(args, w: gen.Workload) -> dict:
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    import deformable_convolution_sampling_b200 as dcn

    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[w.dtype]
    inp = gen.make_inputs(w, tail_fill=0.0)

    def host_tensor(a):
        import numpy as np
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(tdt) if w.dtype == "bf16" else torch.from_numpy(a)
        return t.pin_memory()

    h_v, h_om, h_gy = host_tensor(inp["value"]), host_tensor(inp["offset_mask"]), host_tensor(inp["grad_out"])
    v, om, gy = h_v.to(dev), h_om.to(dev), h_gy.to(dev)
    p = dcn.make_params(dtype=w.dtype, **w.geometry())
    st, Ho, Wo = dcn.dcn4_output_dims(p)
    dcn.check(st)
    out = torch.empty((w.N, Ho, Wo, w.C), dtype=tdt, device=dev)
    gv = torch.empty_like(v)
    gom = torch.empty((w.N, Ho, Wo, w.P), dtype=tdt, device=dev)
    ws_bytes = dcn.dcn4_backward_workspace_size(p)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    ptr = dict(v=v.data_ptr(), om=om.data_ptr(), gy=gy.data_ptr(), out=out.data_ptr(), gv=gv.data_ptr(),
               gom=gom.data_ptr(), ws=ws.data_ptr())

    def fwd():
        dcn.check(dcn.dcn4_forward(p, ptr["v"], ptr["om"], ptr["out"], sh))

    def bwd_om():
        dcn.check(dcn.dcn4_backward_offset_mask(p, ptr["v"], ptr["om"], ptr["gy"], ptr["gom"], ptr["ws"], ws_bytes, sh))

    def bwd_val():
        dcn.check(dcn.dcn4_backward_value(p, ptr["om"], ptr["gy"], ptr["gv"], ptr["ws"], ws_bytes, sh))

    def bwd():
        bwd_om()
        bwd_val()

    stages = [("fwd", fwd), ("bwd_offset_mask", bwd_om), ("bwd_value", bwd_val)]
    launches_per_step = len(stages)  # forward, grad_offset_mask kernel, grad_value kernel (+ a 4N-byte memset)

    for _ in range(args.warmup):
        flush.zero_()
        for _, fn in stages:
            fn()
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(local if world > 1 else torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(K)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    t0 = time.time()
    for i in range(K):
        flush.zero_()
        ev[i][0].record(stream)
        for j, (_, fn) in enumerate(stages):
            fn()
            ev[i][j + 1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    t1 = time.time()
    time.sleep(0.25)
    sampler.stop()

    stage_us = {}
    for j, (name, _) in enumerate(stages):
        stage_us[name] = max_over_ranks(statistics.mean(e[j].elapsed_time(e[j + 1]) for e in ev) * 1e3, dev)
    step_ms = statistics.mean(e[0].elapsed_time(e[-1]) for e in ev)
    step_ms_max = max_over_ranks(step_ms, dev)
    fwd_us = stage_us["fwd"]
    bwd_us = stage_us["bwd_offset_mask"] + stage_us["bwd_value"]

    # End to end through host buffers: every step copies its inputs from pinned
    # host memory, runs forward + backward through the C ABI and copies its three
    # results back to pinned host memory, all inside the timed region.  Steps are
    # pipelined over two sets of device buffers on three streams (copy in,
    # compute, copy out), so one step's results travel back while the next
    # step's inputs travel in and it computes -- PCIe carries both directions at
    # once.  The serial figure (copy in, compute, copy out, one step at a time)
    # is reported beside it.
    e2e = None
    if not args.no_e2e:
        h_out = torch.empty(out.shape, dtype=tdt).pin_memory()
        h_gv = torch.empty(gv.shape, dtype=tdt).pin_memory()
        h_gom = torch.empty(gom.shape, dtype=tdt).pin_memory()
        bi = sum(t.numel() * t.element_size() for t in (h_v, h_om, h_gy))
        bo = sum(t.numel() * t.element_size() for t in (h_out, h_gv, h_gom))
        ke = max(3, min(K, 50))

        def serial_step():
            v.copy_(h_v, non_blocking=True)
            om.copy_(h_om, non_blocking=True)
            gy.copy_(h_gy, non_blocking=True)
            fwd()
            bwd()
            h_out.copy_(out, non_blocking=True)
            h_gv.copy_(gv, non_blocking=True)
            h_gom.copy_(gom, non_blocking=True)

        for _ in range(3):
            serial_step()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dev)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(ke):
            serial_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        serial_us = max_over_ranks(e0.elapsed_time(e1) * 1e3 / ke, dev)

        # second set of device buffers and the three streams
        bufs = [dict(v=v, om=om, gy=gy, out=out, gv=gv, gom=gom),
                dict(v=torch.empty_like(v), om=torch.empty_like(om), gy=torch.empty_like(gy),
                     out=torch.empty_like(out), gv=torch.empty_like(gv), gom=torch.empty_like(gom))]
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e in ev_comp + ev_out:
            e.record(stream)  # both buffer sets start free

        def pipelined_step(i):
            b = i & 1
            d = bufs[b]
            with torch.cuda.stream(s_in):  # inputs of buffer set b are free once its last compute is done
                s_in.wait_event(ev_comp[b])
                d["v"].copy_(h_v, non_blocking=True)
                d["om"].copy_(h_om, non_blocking=True)
                d["gy"].copy_(h_gy, non_blocking=True)
                ev_in[b].record(s_in)
            s_comp.wait_event(ev_in[b])
            s_comp.wait_event(ev_out[b])  # its results have left the device
            cs = s_comp.cuda_stream
            dcn.check(dcn.dcn4_forward(p, d["v"].data_ptr(), d["om"].data_ptr(), d["out"].data_ptr(), cs))
            dcn.check(dcn.dcn4_backward_offset_mask(p, d["v"].data_ptr(), d["om"].data_ptr(), d["gy"].data_ptr(),
                                                    d["gom"].data_ptr(), ws.data_ptr(), ws_bytes, cs))
            dcn.check(dcn.dcn4_backward_value(p, d["om"].data_ptr(), d["gy"].data_ptr(), d["gv"].data_ptr(),
                                              ws.data_ptr(), ws_bytes, cs))  # computes are serial on s_comp
            ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                h_out.copy_(d["out"], non_blocking=True)
                h_gv.copy_(d["gv"], non_blocking=True)
                h_gom.copy_(d["gom"], non_blocking=True)
                ev_out[b].record(s_out)

        for i in range(4):
            pipelined_step(i)
        torch.cuda.synchronize(dev)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dev)
        torch.cuda.synchronize(dev)
        p0.record(s_in)
        for i in range(ke):
            pipelined_step(i)
        s_in.wait_stream(s_out)
        p1.record(s_in)
        torch.cuda.synchronize(dev)
        e2e_us = max_over_ranks(p0.elapsed_time(p1) * 1e3 / ke, dev)
        e2e = {"value": round(e2e_us, 2), "unit": "us/call", "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
               "steps": ke, "pipelined": "2 buffer sets, copy-in / compute / copy-out streams",
               "serial_value": round(serial_us, 2)}

    bm = byte_model(w)
    peaks = measured_peaks()
    fwd_gbs = bm["fwd"] / (fwd_us * 1e-6) / 1e9
    bwd_gbs = bm["bwd"] / (bwd_us * 1e-6) / 1e9
    step_gbs = (bm["fwd"] + bm["bwd"]) / (step_ms_max * 1e-3) / 1e9
    dominant = max(stage_us, key=stage_us.get)
    dom_gbs = bm[dominant] / (stage_us[dominant] * 1e-6) / 1e9
    roofline = {
        "bound": "hbm", "kernel": KERNELS[dominant], "launch_us": round(stage_us[dominant], 2),
        "achieved": round(dom_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": round(dom_gbs / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
        "traffic": recorded_traffic(KERNELS[dominant], w.name),
        "algorithmic_bytes": bm[dominant],
    }

    clocks = summarize_clocks(sampler.samples, t0, t1)
    result = {
        "metric": METRIC, "value": round(step_ms_max * 1e3, 2), "unit": "us/call",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 5),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.describe()}, forward+backward",
                   "global_batch": w.N * world, "parallelism": f"replicas x{world} (batch per GPU {w.N})",
                   "l2": "flushed between timed steps (256 MiB write outside the events)"},
        "fwd_us": round(fwd_us, 2), "bwd_us": round(bwd_us, 2),
        "kernel_us": {KERNELS[k]: round(v, 2) for k, v in stage_us.items()},
        "fwd_gbs": round(fwd_gbs, 1), "bwd_gbs": round(bwd_gbs, 1), "step_gbs": round(step_gbs, 1),
        "fwd_frac_hbm": round(fwd_gbs / peaks["hbm_gbs"], 4), "bwd_frac_hbm": round(bwd_gbs / peaks["hbm_gbs"], 4),
        "fwd_frac_8tbs": round(fwd_gbs / 8000.0, 4), "bwd_frac_8tbs": round(bwd_gbs / 8000.0, 4),
        "bytes_per_call": bm,
        "roofline": roofline,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    if e2e is not None:
        result["e2e"] = e2e
    if not args.no_linear:
        result["linear"] = linear_leg(w, v, gy, p, flush, stream, dev, world)
        result["projection"] = proj_leg(w, v, om, p, flush, stream, dev, world)
    if not args.no_per_config:
        sampler = ClockSampler(local if world > 1 else torch.cuda.current_device())
        sampler.start()
        time.sleep(0.3)
        t2 = time.time()
        result["per_config"] = per_config_leg(dev, world, args.config_reps, flush, stream)
        t3 = time.time()
        sampler.stop()
        result["per_config_clocks"] = summarize_clocks(sampler.samples, t2, t3)
        result["per_config_note"] = (f"{args.config_reps} calls of each stage per workload, CUDA events on the "
                                     f"launching stream, L2 flushed before every call; fractions of the measured "
                                     f"copy bandwidth ({measured_peaks()['hbm_gbs']} GB/s) and of 8 TB/s")
        result["attention"] = attention_leg(dev, world, args.config_reps, flush, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = time_oracle(w, args.cpu_seconds)
    if world > 1:
        dist.destroy_process_group()
    return result


def config_record(w: gen.Workload, stage_us: dict, peaks: dict) -> dict:
    """µs per call and achieved HBM GB/s against the algorithmic byte model."""
    bm = byte_model(w)
    fwd_us = stage_us["fwd"]
    bwd_us = stage_us["bwd_offset_mask"] + stage_us["bwd_value"]
    rec = {"workload": f"{w.name}: {w.describe()}", "fwd_us": round(fwd_us, 2), "bwd_us": round(bwd_us, 2),
           "kernel_us": {KERNELS[k]: round(v, 2) for k, v in stage_us.items()},
           "fwd_bytes": bm["fwd"], "bwd_bytes": bm["bwd"]}
    for leg, us, b in (("fwd", fwd_us, bm["fwd"]), ("bwd", bwd_us, bm["bwd"])):
        gbs = b / (us * 1e-6) / 1e9
        rec[f"{leg}_gbs"] = round(gbs, 1)
        rec[f"{leg}_frac_hbm"] = round(gbs / peaks["hbm_gbs"], 4)
        rec[f"{leg}_frac_8tbs"] = round(gbs / 8000.0, 4)
    return rec


def per_config_leg(dev, world: int, reps: int, flush, stream) -> dict:
    """Every workload of the configuration table: forward, grad_offset_mask and
    grad_value stages, each timed over `reps` calls with CUDA events on the
    launching stream and the L2 flushed before every call (outside the events);
    max over ranks."""
    import numpy as np
    import torch
    import deformable_convolution_sampling_b200 as dcn
    peaks = measured_peaks()
    sh = stream.cuda_stream
    out = {}
    for name in gen.WORKLOAD_ORDER:
        w = gen.WORKLOADS[name]
        tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[w.dtype]
        inp = gen.make_inputs(w, tail_fill=0.0)

        def dev_t(a):
            a = np.ascontiguousarray(a)
            t = torch.from_numpy(a.view(np.int16)).view(tdt) if w.dtype == "bf16" else torch.from_numpy(a)
            return t.to(dev)
        v, om, gy = dev_t(inp["value"]), dev_t(inp["offset_mask"]), dev_t(inp["grad_out"])
        p = dcn.make_params(dtype=w.dtype, **w.geometry())
        y = torch.empty((w.N, w.Ho, w.Wo, w.C), dtype=tdt, device=dev)
        gv, gom = torch.empty_like(v), torch.empty_like(om)
        nb = dcn.dcn4_backward_workspace_size(p)
        ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
        calls = {
            "fwd": lambda: dcn.check(dcn.dcn4_forward(p, v.data_ptr(), om.data_ptr(), y.data_ptr(), sh)),
            "bwd_offset_mask": lambda: dcn.check(dcn.dcn4_backward_offset_mask(
                p, v.data_ptr(), om.data_ptr(), gy.data_ptr(), gom.data_ptr(), ws.data_ptr(), nb, sh)),
            "bwd_value": lambda: dcn.check(dcn.dcn4_backward_value(
                p, om.data_ptr(), gy.data_ptr(), gv.data_ptr(), ws.data_ptr(), nb, sh)),
        }
        for _ in range(5):
            for fn in calls.values():
                fn()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(reps)]
        torch.cuda.synchronize(dev)
        for e in ev:
            flush.zero_()
            e[0].record(stream)
            for j, fn in enumerate(calls.values()):
                fn()
                e[j + 1].record(stream)
        torch.cuda.synchronize(dev)
        stage_us = {k: max_over_ranks(statistics.mean(e[j].elapsed_time(e[j + 1]) for e in ev) * 1e3, dev)
                    for j, k in enumerate(calls)}
        out[name] = config_record(w, stage_us, peaks)
        del v, om, gy, y, gv, gom, ws
    torch.cuda.empty_cache()
    return out


def attn_byte_model(w) -> dict:
    """Compulsory bytes of single-scale deformable attention.  forward: value,
    reference points and offset_logits read, out written; backward: value,
    reference points, offset_logits and grad_out read, grad_value and
    grad_offset_logits written."""
    b = ELEM_BYTES[w.dtype]
    value = w.N * w.H * w.W * w.C * b
    ref = w.N * w.Nq * 8
    ol = w.N * w.Nq * w.P * b
    out = w.N * w.Nq * w.C * b
    return {"fwd": value + ref + ol + out, "bwd": value + ref + ol + out + value + ol}


def attention_leg(dev, world: int, reps: int, flush, stream) -> dict:
    """Single-scale deformable attention on its workloads: forward and backward
    µs per call (CUDA events, L2 flushed before every call), achieved GB/s against
    the byte model, fractions of the measured copy bandwidth and of 8 TB/s."""
    import numpy as np
    import torch
    import deformable_convolution_sampling_b200 as dcn
    peaks = measured_peaks()
    sh = stream.cuda_stream
    res = {}
    for name in gen.ATTN_WORKLOAD_ORDER:
        w = gen.ATTN_WORKLOADS[name]
        tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[w.dtype]
        inp = gen.make_attn_inputs(w, tail_fill=0.0)

        def dev_t(a, keep=False):
            a = np.ascontiguousarray(a)
            t = torch.from_numpy(a.view(np.int16)).view(tdt) if (w.dtype == "bf16" and not keep) else torch.from_numpy(a)
            return t.to(dev)
        v, ol, gy = dev_t(inp["value"]), dev_t(inp["offset_logits"]), dev_t(inp["grad_out"])
        ref = dev_t(inp["ref_points"], keep=True)
        p = dcn.make_attn_params(dtype=w.dtype, **w.geometry())
        y = torch.empty((w.N, w.Nq, w.C), dtype=tdt, device=dev)
        gv, gol = torch.empty_like(v), torch.empty_like(ol)
        nb = dcn.dcn4_attn_backward_workspace_size(p)
        ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
        calls = {
            "fwd": lambda: dcn.check(dcn.dcn4_attn_forward(p, v.data_ptr(), ref.data_ptr(), ol.data_ptr(),
                                                           y.data_ptr(), sh)),
            "bwd": lambda: dcn.check(dcn.dcn4_attn_backward(p, v.data_ptr(), ref.data_ptr(), ol.data_ptr(),
                                                            gy.data_ptr(), gv.data_ptr(), gol.data_ptr(),
                                                            ws.data_ptr(), nb, sh)),
        }
        bm = attn_byte_model(w)
        rec = {"workload": f"{w.name}: {w.describe()}"}
        for leg, fn in calls.items():
            for _ in range(5):
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            for e0, e1 in ev:
                flush.zero_()
                e0.record(stream)
                fn()
                e1.record(stream)
            torch.cuda.synchronize(dev)
            us = max_over_ranks(statistics.mean(a.elapsed_time(c) for a, c in ev) * 1e3, dev)
            gbs = bm[leg] / (us * 1e-6) / 1e9
            rec[f"{leg}_us"] = round(us, 2)
            rec[f"{leg}_bytes"] = bm[leg]
            rec[f"{leg}_gbs"] = round(gbs, 1)
            rec[f"{leg}_frac_hbm"] = round(gbs / peaks["hbm_gbs"], 4)
            rec[f"{leg}_frac_8tbs"] = round(gbs / 8000.0, 4)
        res[name] = rec
        del v, ol, gy, ref, y, gv, gol, ws
    torch.cuda.empty_cache()
    return res


def linear_leg(w: gen.Workload, v, gy, p, flush, stream, dev, world: int) -> dict:
    """µs per call (CUDA events, L2 flushed before each, max over ranks): the fused
    forward with and without storing its offset_mask, against cuBLAS's linear layer
    followed by dcn4_forward, on seeded x [N,Ho,Wo,C], W [P,C], b [P]; and the
    layer's backward (dcn4_backward_linear) against dcn4_backward followed by
    cuBLAS products for the linear layer's gradients."""
    import numpy as np
    import torch
    import torch.nn.functional as F
    import deformable_convolution_sampling_b200 as dcn
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16}.get(w.dtype)
    if tdt is None:
        return {"unavailable": "the fused producer takes fp16 or bf16"}
    lin = gen.make_linear_inputs(w, w.C)

    def dev_t(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(tdt) if w.dtype == "bf16" else torch.from_numpy(a)
        return t.to(dev)
    x, wt, b = dev_t(lin["x"]), dev_t(lin["weight"]), dev_t(lin["bias"])
    out = torch.empty((w.N, w.Ho, w.Wo, w.C), dtype=tdt, device=dev)
    om = torch.empty((w.N, w.Ho, w.Wo, w.P), dtype=tdt, device=dev)
    sh = stream.cuda_stream
    ptr = dict(v=v.data_ptr(), x=x.data_ptr(), w=wt.data_ptr(), b=b.data_ptr(), out=out.data_ptr(),
               om=om.data_ptr())

    def fused():
        dcn.check(dcn.dcn4_forward_linear(p, w.C, ptr["v"], ptr["x"], ptr["w"], ptr["b"], ptr["out"], None, sh))

    def fused_om():
        dcn.check(dcn.dcn4_forward_linear(p, w.C, ptr["v"], ptr["x"], ptr["w"], ptr["b"], ptr["out"], ptr["om"], sh))

    def unfused():
        torch.addmm(b, x.view(-1, w.C), wt.t(), out=om.view(-1, w.P))
        dcn.check(dcn.dcn4_forward(p, ptr["v"], ptr["om"], ptr["out"], sh))

    def linear_only():
        torch.addmm(b, x.view(-1, w.C), wt.t(), out=om.view(-1, w.P))

    res = {}
    for name, fn in (("fused_us", fused), ("fused_with_offset_mask_out_us", fused_om),
                     ("cublas_linear_then_forward_us", unfused), ("cublas_linear_us", linear_only)):
        for _ in range(5):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(100)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = round(max_over_ranks(statistics.mean(a.elapsed_time(c) for a, c in ev) * 1e3, dev), 2)
    res["speedup_vs_unfused"] = round(res["cublas_linear_then_forward_us"] / res["fused_us"], 3)
    res["gemm"] = (f"x [{w.N * w.Ho * w.Wo}, {w.C}] @ W^T [{w.C}, {w.P}] + b per 64-pixel tile: tcgen05.mma kind::f16 "
                   f"(M = 128 rows of W, N = 64 pixels, fp32 accumulator in tensor memory) where W fits 128 rows and "
                   f"Cx is 64 or 128, else mma.sync m16n8k16")
    res["launches_per_call"] = 1

    # Backward of the layer: dcn4_backward_linear (the aggregation's backward, then the
    # linear layer's gradients in libdcn4) against dcn4_backward followed by cuBLAS.
    gv, gom = torch.empty_like(v), torch.empty_like(om)
    gx, gw, gb = torch.empty_like(x), torch.empty_like(wt), torch.empty_like(b)
    nb = dcn.dcn4_backward_workspace_size(p)
    nbl = dcn.dcn4_backward_linear_workspace_size(p, w.C)
    ws = torch.empty(max(nbl, 16), dtype=torch.uint8, device=dev)
    fused_om()
    torch.cuda.synchronize(dev)
    g2, x2 = gom.view(-1, w.P), x.view(-1, w.C)

    def bwd_chain():
        dcn.check(dcn.dcn4_backward_linear(p, w.C, ptr["v"], ptr["om"], ptr["x"], ptr["w"], gy.data_ptr(),
                                           gv.data_ptr(), gom.data_ptr(), gx.data_ptr(), gw.data_ptr(), gb.data_ptr(),
                                           ws.data_ptr(), nbl, sh))

    def bwd_only():
        dcn.check(dcn.dcn4_backward(p, ptr["v"], ptr["om"], gy.data_ptr(), gv.data_ptr(), gom.data_ptr(),
                                    ws.data_ptr(), nb, sh))

    def bwd_then_cublas():
        bwd_only()
        torch.mm(g2, wt, out=gx.view(-1, w.C))
        torch.mm(g2.t(), x2, out=gw)
        torch.sum(g2, 0, out=gb)

    for name, fn in (("backward_linear_us", bwd_chain), ("backward_us", bwd_only),
                     ("backward_then_cublas_us", bwd_then_cublas)):
        for _ in range(5):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(100)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = round(max_over_ranks(statistics.mean(a.elapsed_time(c) for a, c in ev) * 1e3, dev), 2)
    M = w.N * w.Ho * w.Wo
    lin_us = res["backward_linear_us"] - res["backward_us"]
    res["linear_backward_us"] = round(lin_us, 2)
    res["cublas_linear_backward_us"] = round(res["backward_then_cublas_us"] - res["backward_us"], 2)
    # g, x read once and grad_x written once: the least the layer's gradients move
    lin_bytes = M * (w.P + 2 * w.C) * 2
    res["linear_backward_bytes"] = lin_bytes
    res["linear_backward_gemm"] = (f"grad_x = g W ([{M}, {w.P}] x [{w.P}, {w.C}]), grad_W = g^T x, grad_b: tcgen05.mma "
                                   f"kind::f16 from TMA-fed 128-byte-swizzled shared memory, fp32 accumulators in "
                                   f"tensor memory, warp-specialised")
    if lin_us > 0:
        res["linear_backward_gbs"] = round(lin_bytes / (lin_us * 1e-6) / 1e9, 1)
    del gv, gom, gx, gw, gb, ws
    return res


def proj_leg(w: gen.Workload, v, om, p, flush, stream, dev, world: int) -> dict:
    """µs per call (CUDA events, L2 flushed before each, max over ranks): the forward
    with the output projection fused behind it (dcn4_forward_proj, Cout = C), with and
    without storing the core output, against dcn4_forward followed by cuBLAS's linear
    layer; and dcn4_backward_proj against cuBLAS products for the projection's
    gradients followed by dcn4_backward."""
    import numpy as np
    import torch
    import deformable_convolution_sampling_b200 as dcn
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16}.get(w.dtype)
    if tdt is None:
        return {"unavailable": "the fused projection takes fp16 or bf16"}
    Cout = w.C
    if dcn.dcn4_forward_proj(p, Cout, None, None, None, None, None) == -5:
        return {"unavailable": dcn.dcn4_last_error()}
    pj = gen.make_proj_inputs(w, Cout)

    def dev_t(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(tdt) if w.dtype == "bf16" else torch.from_numpy(a)
        return t.to(dev)
    wt, b, gy = dev_t(pj["weight"]), dev_t(pj["bias"]), dev_t(pj["grad_out"])
    M = w.N * w.Ho * w.Wo
    core = torch.empty((w.N, w.Ho, w.Wo, w.C), dtype=tdt, device=dev)
    y = torch.empty((w.N, w.Ho, w.Wo, Cout), dtype=tdt, device=dev)
    sh = stream.cuda_stream

    def fused():
        dcn.check(dcn.dcn4_forward_proj(p, Cout, v.data_ptr(), om.data_ptr(), wt.data_ptr(), b.data_ptr(),
                                        y.data_ptr(), None, sh))

    def fused_core():
        dcn.check(dcn.dcn4_forward_proj(p, Cout, v.data_ptr(), om.data_ptr(), wt.data_ptr(), b.data_ptr(),
                                        y.data_ptr(), core.data_ptr(), sh))

    def unfused():
        dcn.check(dcn.dcn4_forward(p, v.data_ptr(), om.data_ptr(), core.data_ptr(), sh))
        torch.addmm(b, core.view(-1, w.C), wt.t(), out=y.view(-1, Cout))

    def linear_only():
        torch.addmm(b, core.view(-1, w.C), wt.t(), out=y.view(-1, Cout))

    gv, gom = torch.empty_like(v), torch.empty_like(om)
    gw, gb, gcore = torch.empty_like(wt), torch.empty_like(b), torch.empty_like(core)
    nb = dcn.dcn4_backward_workspace_size(p)
    nbp = dcn.dcn4_backward_proj_workspace_size(p, Cout)
    ws = torch.empty(max(nbp, 16), dtype=torch.uint8, device=dev)
    g2 = gy.view(-1, Cout)

    def bwd_fused():
        dcn.check(dcn.dcn4_backward_proj(p, Cout, v.data_ptr(), om.data_ptr(), core.data_ptr(), wt.data_ptr(),
                                         gy.data_ptr(), gv.data_ptr(), gom.data_ptr(), gw.data_ptr(), gb.data_ptr(),
                                         ws.data_ptr(), nbp, sh))

    def bwd_only():
        dcn.check(dcn.dcn4_backward(p, v.data_ptr(), om.data_ptr(), gcore.data_ptr(), gv.data_ptr(), gom.data_ptr(),
                                    ws.data_ptr(), nb, sh))

    def cublas_then_bwd():
        torch.mm(g2, wt, out=gcore.view(-1, w.C))
        torch.mm(g2.t(), core.view(-1, w.C), out=gw)
        torch.sum(g2, 0, out=gb)
        bwd_only()

    res = {}
    fused_core()
    torch.cuda.synchronize(dev)
    for name, fn in (("fused_us", fused), ("fused_with_core_out_us", fused_core),
                     ("forward_then_cublas_us", unfused), ("cublas_linear_us", linear_only),
                     ("backward_proj_us", bwd_fused), ("backward_us", bwd_only),
                     ("cublas_then_backward_us", cublas_then_bwd)):
        for _ in range(5):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(100)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = round(max_over_ranks(statistics.mean(a.elapsed_time(c) for a, c in ev) * 1e3, dev), 2)
    res["speedup_vs_unfused"] = round(res["forward_then_cublas_us"] / res["fused_us"], 3)
    res["backward_speedup_vs_unfused"] = round(res["cublas_then_backward_us"] / res["backward_proj_us"], 3)
    res["gemm"] = (f"core [{M}, {w.C}] @ W^T [{w.C}, {Cout}] + b per tile: tcgen05.mma kind::f16 (M = 128 rows of W, "
                   f"N = the tile's pixels, fp32 accumulator in tensor memory), core rows written to shared memory by "
                   f"the sampling threads")
    res["launches_per_call"] = 1
    res["projection_backward_us"] = round(res["backward_proj_us"] - res["backward_us"], 2)
    res["cublas_projection_backward_us"] = round(res["cublas_then_backward_us"] - res["backward_us"], 2)
    del gv, gom, gw, gb, gcore, ws, core, y
    return res


def run_profile(args, w: gen.Workload) -> None:
    """--profile: warm-up + steps passes of the path (forward and backward of the
    workload; with --linear the fused forward and dcn4_backward_linear too; with
    --proj the forward with its fused output projection and dcn4_backward_proj)
    with no timing and no JSON line -- a short, fixed launch sequence for ncu
    captures."""
    import numpy as np
    import torch
    import deformable_convolution_sampling_b200 as dcn
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[w.dtype]

    def dev_t(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(tdt) if w.dtype == "bf16" else torch.from_numpy(a)
        return t.to(dev)
    inp = gen.make_inputs(w, tail_fill=0.0)
    v, om, gy = dev_t(inp["value"]), dev_t(inp["offset_mask"]), dev_t(inp["grad_out"])
    p = dcn.make_params(dtype=w.dtype, **w.geometry())
    lin = None
    if args.linear:
        li = gen.make_linear_inputs(w, w.C)
        lin = dev_t(li["x"]), dev_t(li["weight"]), dev_t(li["bias"])
    proj = None
    if args.proj:
        pj = gen.make_proj_inputs(w, w.C)
        proj = dev_t(pj["weight"]), dev_t(pj["bias"]), dev_t(pj["grad_out"])
    for _ in range(args.warmup + args.steps):
        dcn.forward(p, v, om)
        dcn.backward(p, v, om, gy)
        if lin is not None:
            om_lin = torch.empty_like(om)
            dcn.forward_linear(p, v, *lin, offset_mask_out=om_lin)
            dcn.backward_linear(p, v, om_lin, lin[0], lin[1], gy)
        if proj is not None:
            core = torch.empty((w.N, w.Ho, w.Wo, w.C), dtype=tdt, device=dev)
            dcn.forward_proj(p, v, om, proj[0], proj[1], core_out=core)
            dcn.backward_proj(p, v, om, core, proj[0], proj[2])
    torch.cuda.synchronize(dev)
    print(f"profile: {w.name}: {args.warmup + args.steps} passes done", flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="stage1_f16", choices=sorted(gen.WORKLOADS))
    ap.add_argument("--softmax", action="store_true",
                    help="masks are logits normalised by a softmax over the K points (DCNv3 form)")
    ap.add_argument("--no-linear", action="store_true",
                    help="skip the timings of the layer with its offset/mask linear producer (fused forward, "
                         "dcn4_backward_linear)")
    ap.add_argument("--linear", action="store_true",
                    help="with --profile: also run the fused forward and dcn4_backward_linear")
    ap.add_argument("--proj", action="store_true",
                    help="with --profile: also run the forward with its fused output projection and "
                         "dcn4_backward_proj")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-workload forward/backward timings")
    ap.add_argument("--config-reps", type=int, default=50,
                    help="calls per stage and workload in the per-config timings")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--profile", action="store_true",
                    help="run warm-up + steps untimed passes of --workload for an ncu capture; no JSON line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = gen.WORKLOADS[args.workload]
    if args.softmax:
        w = dataclasses.replace(w, softmax=1, name=w.name + "_softmax")
    if args.profile:
        run_profile(args, w)
        return
    rank, world, _ = dist_env()
    if args.impl == "reference":
        res = run_reference(args, w)
    else:
        res = run_native(args, w)
    if rank == 0 and res:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
