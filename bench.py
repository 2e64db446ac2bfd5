"""Benchmark of the exact-attention hot path on B200: one step = fa2_fwd + fa2_bwd.

The default step is the training shape B=8, H=16, N=4096, d=128, bf16, causal (the
largest forward + backward workload that fits one GPU; inputs x0.5).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-extras]

Prints ONE JSON line on rank 0.  ``value`` is whole-job TFLOP/s of the algorithmic
FLOPs (forward 4 B H N^2 d, halved when causal; backward 2.5x forward) over the
device time of exactly K timed steps (CUDA events on the launching stream, max over
ranks).  Inputs are seeded synthetic tensors already resident in HBM; when they fit
in L2 a 256 MiB buffer is written between steps (outside the events) to flush it.

Multi-GPU (under torchrun): every rank runs an independent replica of the same
workload (the attention of every (batch, head) is independent; no collective sits
on the data path), so scaling is weak.

``--impl reference`` times the CPU fp64 oracle (the reference arm)
on a bounded sample of the same workload, on rank 0 only.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from exact_io_aware_74_b200.workloads import (  # noqa: E402
    DECODE_WORKLOADS, FP8_WORKLOADS, WORKLOADS, WORKLOAD_ORDER, decode_inputs, make_fp8_inputs,
    workload_inputs)

METRIC = "FA-2 fwd/bwd TFLOP/s (bf16, 1×B200) and % of dense BF16 tensor peak"
DEFAULT_WORKLOAD = "fwdbwd_bf16_b8h16_n4096_d128_causal"  # forward + backward, the training shape
HEADLINE_WORKLOAD = WORKLOAD_ORDER[2]         # forward, bf16, non-causal, N = 8192, d = 128
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------------
# helpers (host logic; tested on CPU)
# ------------------------------------------------------------------------------------

def load_peaks(path: str | None = None) -> tuple[dict, str]:
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            data = json.load(f)
        return {k: float(data[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def step_flops(w) -> float:
    return w.fwd_flops + (w.bwd_flops if w.backward else 0.0)


# NVIDIA's published dense (no 2:4 sparsity) bf16 tensor throughput of one B200.
DATASHEET_BF16_TFLOPS = 2250.0


def fwd_bytes(w) -> int:
    """Algorithmic HBM bytes of one forward: Q, K, V read once, O written once (16-bit),
    LSE written (fp32)."""
    return w.B * w.H * w.N * (4 * w.d * 2 + 4)


def bwd_bytes(w) -> int:
    """Algorithmic HBM bytes of one backward: Q, K, V, O, dO read and dQ, dK, dV written
    once (16-bit), LSE read (fp32)."""
    return w.B * w.H * w.N * (8 * w.d * 2 + 4)


def input_bytes(w) -> int:
    n = w.B * w.H * w.N * w.d * 2
    return n * (4 if w.backward else 3)


# Device sources of each C-ABI call's kernels.
KERNEL_SOURCES = {"fa2_fwd": ("ptx.cuh", "fa2_fwd.cuh"),
                  "fa2_bwd": ("ptx.cuh", "fa2_bwd.cuh", "fa2_bwd_dq.cuh"),
                  "fa2_fwd_decode": ("ptx.cuh", "fa2_fwd.cuh", "fa2_decode.cuh")}


def _code_only(src: str) -> str:
    """C++ source without comments and blank lines: edits to comments alone do not
    change the kernels a traffic record was taken from."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = []
    for line in src.splitlines():
        # drop // comments (the kernels have no "//" inside string literals)
        line = line.split("//", 1)[0].rstrip()
        if line:
            out.append(line)
    return "\n".join(out)


def csrc_hash(call: str) -> str:
    """Hash of the code (comments aside) of the device source files of one call's kernels."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_74_b200", "csrc")
    for name in KERNEL_SOURCES[call]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_from_profiles(kernel_key: str) -> int | None:
    """DRAM bytes per call recorded by an ncu capture of the current kernel source.

    ``profiles/dram_traffic.txt`` holds lines ``<call>:<workload> <source hash>
    <bytes>``; a record taken from another version of the kernels does not count.
    """
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    cur = csrc_hash(kernel_key.split(":")[0])
    for ln in lines:
        parts = ln.split()
        if len(parts) == 3 and parts[0] == kernel_key and parts[1] == cur:
            return int(float(parts[2]))
    return None


def aggregate(local_time_s: float, local_flops: float, world: int) -> tuple[float, float]:
    """(max time over ranks, total FLOPs over ranks); identity without a process group."""
    if world <= 1 or not torch.distributed.is_initialized():
        return local_time_s, local_flops
    backend = torch.distributed.get_backend()
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else "cpu"
    t = torch.tensor([local_time_s], dtype=torch.float64, device=dev)
    f = torch.tensor([local_flops], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.all_reduce(f, op=torch.distributed.ReduceOp.SUM)
    return float(t.item()), float(f.item())


class ClockSampler:
    """Samples SM clock, power and clock-event reasons with NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the host (NVML present or not)
            self.error = repr(e)
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        nv, h = self._nv, self._h
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                reasons = int(get_reasons(h)) if get_reasons else 0
                self.samples.append((mhz, reasons))
            except Exception as e:  # pragma: no cover
                self.error = repr(e)
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "error": self.error}
        mhz = [s for s, _ in self.samples]
        seen = 0
        for _, r in self.samples:
            seen |= r
        names = [n for bit, n in self.REASONS.items() if seen & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(mhz)}


# ------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------

def _fa2():
    from exact_io_aware_74_b200 import fa2
    fa2.load()  # raises if the CUDA library is missing: there is no fallback
    return fa2


def _check(fa2, rc, what):
    if rc != fa2.FA2_OK:
        raise RuntimeError(f"{what}: {fa2.status_string(rc)}")


class Step:
    """Device buffers and the two C-ABI calls of one step of a workload.  ``host``
    (pinned host inputs) may be shared with another Step: a second set of device
    buffers for the same inputs."""

    def __init__(self, fa2, w, dev, host=None):
        self.fa2, self.w = fa2, w
        if host is None:
            x = workload_inputs(w)
            host = {k: x[k].pin_memory() for k in ("q", "k", "v", "do") if k in x}
        self.host = host
        self.q, self.k, self.v = (self.host[n].to(dev) for n in ("q", "k", "v"))
        self.do = self.host["do"].to(dev) if w.backward else None
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        if w.backward:
            self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
            self.ws = torch.empty(fa2.fa2_bwd_workspace_size(w.B, w.H, w.N, w.d),
                                  dtype=torch.uint8, device=dev)

    def fwd(self, stream):
        if self.w.window:
            rc = self.fa2.fa2_fwd_window(self.q, self.k, self.v, self.o, self.lse, self.w.scale,
                                         self.w.window, stream)
        else:
            rc = self.fa2.fa2_fwd(self.q, self.k, self.v, self.o, self.lse, self.w.scale,
                                  self.w.causal, stream)
        _check(self.fa2, rc, "fa2_fwd")

    def bwd(self, stream):
        if self.w.window:
            rc = self.fa2.fa2_bwd_window(self.q, self.k, self.v, self.o, self.do, self.lse,
                                         self.dq, self.dk, self.dv, self.ws, self.w.scale,
                                         self.w.window, stream)
        else:
            rc = self.fa2.fa2_bwd(self.q, self.k, self.v, self.o, self.do, self.lse, self.dq,
                                  self.dk, self.dv, self.ws, self.w.scale, self.w.causal, stream)
        _check(self.fa2, rc, "fa2_bwd")

    def results(self):
        return (self.dq, self.dk, self.dv) if self.w.backward else (self.o, self.lse)


def time_workload(fa2, w, steps, warmup, dev, stream, flush=None, sampler=None):
    """Per-call CUDA-event timing of K steps; returns per-call millisecond lists."""
    st = Step(fa2, w, dev)
    for _ in range(warmup):
        st.fwd(stream)
        if w.backward:
            st.bwd(stream)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    if torch.distributed.is_initialized():
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = fa2.fa2_launch_count()
    with torch.cuda.stream(stream):
        for i in range(steps):
            if flush is not None:
                flush.add_(1)
            ev[i][0].record(stream)
            st.fwd(stream)
            ev[i][1].record(stream)
            if w.backward:
                st.bwd(stream)
            ev[i][2].record(stream)
    torch.cuda.synchronize()
    if torch.distributed.is_initialized():
        torch.distributed.barrier()
    launches = fa2.fa2_launch_count() - launches0
    rc, site = fa2.fa2_get_device_status(stream)
    if rc != fa2.FA2_OK:
        raise RuntimeError(f"device status {fa2.status_string(rc)} at wait site {site}")
    fwd_ms = [e[0].elapsed_time(e[1]) for e in ev]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in ev] if w.backward else []
    return st, fwd_ms, bwd_ms, launches


def time_e2e(fa2, st, steps, stream):
    """The same step through the public calls, with each step's inputs copied from
    pinned host memory and its results read back, all inside the timed region.

    Pipelined as a user's training or inference loop would be: two sets of device
    buffers, host-to-device copies on one stream, the C-ABI calls on ``stream``,
    device-to-host copies on a third, so that step k+1's upload and step k-1's
    download overlap step k's kernels.  Events order the buffer reuse.
    """
    w = st.w
    dev = st.q.device
    sets = [st, Step(fa2, w, dev, host=st.host)]
    names = [n for n in ("q", "k", "v", "do") if n in st.host]
    outs = [s.results() for s in sets]
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in o] for o in outs]
    h2d = sum(st.host[n].numel() * st.host[n].element_size() for n in names)
    d2h = sum(t.numel() * t.element_size() for t in outs[0])
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)
    in_done = [ev(), ev()]
    computed = [ev(), ev()]
    out_done = [ev(), ev()]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s_in)
    for k in range(steps):
        b = k % 2
        cur = sets[b]
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(computed[b])  # set b's inputs are free again
            for n in names:
                getattr(cur, n).copy_(cur.host[n], non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(in_done[b])
            if k >= 2:
                stream.wait_event(out_done[b])  # set b's results were read back
            cur.fwd(stream)
            if w.backward:
                cur.bwd(stream)
            computed[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[b])
            for h, t in zip(host_out[b], outs[b]):
                h.copy_(t, non_blocking=True)
            out_done[b].record(s_out)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return ms, h2d, d2h


def time_decode(fa2, w, iters, dev, stream, hbm_peak, peaks_src):
    """One decode-like call (fa2_fwd_decode, the library's split count) per step:
    median CUDA-event time, achieved algorithmic HBM GB/s and its roofline."""
    x = decode_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    splits = fa2.fa2_fwd_decode_splits(w.B, w.H, w.Nq, w.Nk, w.d)
    if splits < 1:
        raise RuntimeError("fa2_fwd_decode_splits failed")
    nws = fa2.fa2_fwd_decode_workspace_size(w.B, w.H, w.Nq, w.Nk, w.d, splits)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev) if nws else None
    flush = None
    if w.hbm_bytes < 2 * L2_BYTES:
        flush = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def call():
        _check(fa2, fa2.fa2_fwd_decode(q, k, v, o, lse, w.scale, w.causal, splits, ws, stream),
               "fa2_fwd_decode")

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
    c0 = fa2.fa2_launch_count()
    with torch.cuda.stream(stream):
        for i in range(iters):
            if flush is not None:
                flush.add_(1)
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    launches = (fa2.fa2_launch_count() - c0) // iters
    rc, site = fa2.fa2_get_device_status(stream)
    if rc != fa2.FA2_OK:
        raise RuntimeError(f"device status {fa2.status_string(rc)} at wait site {site}")
    ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    gbs = w.hbm_bytes / (ms / 1e3) / 1e9
    return {"us": round(ms * 1e3, 2), "splits": splits, "launches_per_call": launches,
            "hbm_bytes": w.hbm_bytes, "tflops": round(w.fwd_flops / ms / 1e9, 2),
            "roofline": {"bound": "hbm", "kernel": "fa2_fwd_decode (forward + merge)",
                         "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4),
                         "traffic": traffic_from_profiles(f"fa2_fwd_decode:{w.name}"),
                         "peak_kind": f"HBM copy, {peaks_src}"}}


# Nominal dense 8-bit / 16-bit tensor throughput on B200 (4.5 / 2.25 PFLOP/s): the
# 8-bit roofline is the measured 16-bit peak times this ratio.
FP8_OVER_BF16 = 2.0


def time_fp8(fa2, w, iters, dev, stream, bf16_peak, peaks_src):
    """fa2_fwd_fp8 on an E4M3 workload: median CUDA-event time per call, algorithmic
    TFLOP/s and the fraction of the 8-bit tensor peak."""
    x = make_fp8_inputs(w.B, w.H, w.N, w.d, seed=w.seed)
    s = x["scale"]
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)

    def call():
        _check(fa2, fa2.fa2_fwd_fp8(q, k, v, o, lse, w.scale, w.causal, s, s, s, stream),
               "fa2_fwd_fp8")

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(iters)]
    with torch.cuda.stream(stream):
        for i in range(iters):
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    rc, site = fa2.fa2_get_device_status(stream)
    if rc != fa2.FA2_OK:
        raise RuntimeError(f"device status {fa2.status_string(rc)} at wait site {site}")
    ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    tf = w.fwd_flops / ms / 1e9
    peak = bf16_peak * FP8_OVER_BF16
    return {"fwd_ms": round(ms, 4), "fwd_tflops": round(tf, 1),
            "roofline": {"bound": "tensor", "kernel": "fa2_fwd_kernel (E4M3)",
                         "achieved": round(tf, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tf / peak, 4),
                         "peak_kind": f"bf16 burst x {FP8_OVER_BF16} (nominal e4m3/bf16), "
                                      f"{peaks_src}"}}


def cpu_baseline(w, budget_s: float = 12.0) -> dict:
    """The oracle as it stands, timed on this host's cores on whole (b, h) slices."""
    import numpy as np  # noqa: F401
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        cores = len(os.sched_getaffinity(0))
    x = workload_inputs(w, B=1, H=1)
    per_head = w.fwd_flops / (w.B * w.H) + (w.bwd_flops / (w.B * w.H) if w.backward else 0.0)
    done, t0 = 0, time.perf_counter()
    win = w.window or None
    while True:
        oracle.attn_fwd_ref(x["q"], x["k"], x["v"], w.scale, w.causal, window=win)
        if w.backward:
            oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, window=win)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= w.B * w.H:
            break
    return {"value": round(per_head * done / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{done} of {w.B * w.H} (batch, head) slices of {w.name} "
                      f"({'fwd+bwd' if w.backward else 'fwd'}), fp64 NumPy, {el:.1f} s"}


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    fa2 = _fa2()
    peaks, peaks_src = load_peaks()
    w = WORKLOADS[args.workload]
    stream = torch.cuda.Stream(device=dev)
    flush = None
    if input_bytes(w) * 2 < 2 * L2_BYTES:
        flush = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    with sampler:
        st, fwd_ms, bwd_ms, launches = time_workload(fa2, w, args.steps, args.warmup, dev, stream,
                                                     flush)
    step_ms = [a + b for a, b in zip(fwd_ms, bwd_ms or [0.0] * len(fwd_ms))]
    total_s, total_flops = aggregate(sum(step_ms) / 1e3, step_flops(w) * args.steps, world)
    value = total_flops / total_s / 1e12
    # Dominant call of the step and its roofline.  Each call is timed on its own
    # (CUDA events around it, milliseconds long), so the peak is the burst figure.
    calls = {"fa2_fwd": (statistics.mean(fwd_ms), w.fwd_flops, "fa2_fwd_kernel")}
    if w.backward:
        calls["fa2_bwd"] = (statistics.mean(bwd_ms), w.bwd_flops, "fa2_bwd (pre+main+dq)")
    dom = max(calls, key=lambda k: calls[k][0])
    dom_ms, dom_flops, dom_label = calls[dom]
    achieved = dom_flops / (dom_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    traffic = traffic_from_profiles(f"{dom}:{w.name}")
    e2e_steps = max(1, min(args.steps, 30))
    e2e_ms, h2d, d2h = time_e2e(fa2, st, e2e_steps, stream)
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_s * 1e3 / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "step": "fa2_fwd + fa2_bwd" if w.backward else "fa2_fwd",
                   "l2": ("256 MiB buffer written between steps (outside the timed events)"
                          if flush is not None else "inputs larger than L2"),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "pct_of_peak": {"bf16_burst": round(100 * value / world / peaks["bf16_tflops"], 1),
                        "bf16_sustained": round(100 * value / world / peaks["bf16_tflops_sustained"], 1),
                        "datasheet_dense_bf16": round(100 * value / world / DATASHEET_BF16_TFLOPS, 1),
                        "source": peaks_src},
        "calls_gbs": {"fa2_fwd": round(fwd_bytes(w) / statistics.mean(fwd_ms) / 1e6, 1),
                      **({"fa2_bwd": round(bwd_bytes(w) / statistics.mean(bwd_ms) / 1e6, 1)}
                         if w.backward else {})},
        "calls_ms": {k: round(v[0], 5) for k, v in calls.items()},
        "roofline": {"bound": "tensor", "kernel": dom_label, "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic,
                     "peak_kind": f"bf16 burst, {peaks_src}"},
        "e2e": {"value": round(step_flops(w) / (e2e_ms / 1e3) / 1e12 * world, 3),
                "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps,
                "pipeline": "two buffer sets; uploads, kernels and downloads on three streams"},
        "gpu_launches": launches,
        "clocks": sampler.summary(),
    }
    if not args.no_extras and rank == 0:
        extras = {}
        # every workload but the small fp16 forward (below) and the bench step itself
        for name in [n for n in WORKLOAD_ORDER[1:] if n != w.name]:
            ww = WORKLOADS[name]
            _, f_ms, b_ms, _ = time_workload(fa2, ww, 20, 3, dev, stream, None)
            fm = statistics.median(f_ms)
            e = {"fwd_ms": round(fm, 4), "fwd_tflops": round(ww.fwd_flops / fm / 1e9, 1),
                 "fwd_pct_bf16_burst": round(100 * ww.fwd_flops / fm / 1e9 / peaks["bf16_tflops"], 1),
                 "fwd_pct_bf16_sustained": round(
                     100 * ww.fwd_flops / fm / 1e9 / peaks["bf16_tflops_sustained"], 1),
                 "fwd_pct_datasheet": round(100 * ww.fwd_flops / fm / 1e9 / DATASHEET_BF16_TFLOPS, 1),
                 "fwd_gbs": round(fwd_bytes(ww) / fm / 1e6, 1)}
            if ww.backward:
                bm = statistics.median(b_ms)
                e.update({"bwd_ms": round(bm, 4), "bwd_tflops": round(ww.bwd_flops / bm / 1e9, 1),
                          "bwd_pct_bf16_burst": round(
                              100 * ww.bwd_flops / bm / 1e9 / peaks["bf16_tflops"], 1),
                          "bwd_gbs": round(bwd_bytes(ww) / bm / 1e6, 1)})
            extras[name] = e
            torch.cuda.empty_cache()
        # The small fp16 forward is latency-bound: microseconds and bytes per second.
        w1 = WORKLOADS[WORKLOAD_ORDER[0]]
        flush1 = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        _, f_ms, _, _ = time_workload(fa2, w1, 50, 5, dev, stream, flush1)
        fm = statistics.median(f_ms)
        out["small"] = {"workload": w1.name, "fwd_us": round(fm * 1e3, 2),
                        "fwd_gbs": round(fwd_bytes(w1) / fm / 1e6, 1),
                        "fwd_tflops": round(w1.fwd_flops / fm / 1e9, 3),
                        "note": "launch/latency-bound: 129 KiB of traffic, one CTA per head"}
        del flush1
        out["other_workloads"] = extras
        out["decode"] = {name: time_decode(fa2, dw, 50, dev, stream, peaks["hbm_gbs"], peaks_src)
                         for name, dw in DECODE_WORKLOADS.items()}
        out["fp8"] = {name: time_fp8(fa2, fw, 20, dev, stream, peaks["bf16_tflops"], peaks_src)
                      for name, fw in FP8_WORKLOADS.items()}
        torch.cuda.empty_cache()
        out["headline"] = {"workload": HEADLINE_WORKLOAD,
                           "fwd_tflops": extras[HEADLINE_WORKLOAD]["fwd_tflops"],
                           "pct_of_bf16_burst_peak": extras[HEADLINE_WORKLOAD]["fwd_pct_bf16_burst"],
                           "pct_of_bf16_sustained_peak":
                               extras[HEADLINE_WORKLOAD]["fwd_pct_bf16_sustained"],
                           "pct_of_datasheet_dense_bf16": extras[HEADLINE_WORKLOAD]["fwd_pct_datasheet"],
                           "target_pct": 60.0}
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        line = json.dumps(out)
        print(line, flush=True)
        if args.json_out:
            with open(args.json_out, "w") as f:
                f.write(line + "\n")
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------------------------------
# reference arm: the CPU oracle
# ------------------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    w = WORKLOADS[args.workload]
    x = workload_inputs(w, B=1, H=1)
    per_head = step_flops(w) / (w.B * w.H)

    win = w.window or None

    def one():
        oracle.attn_fwd_ref(x["q"], x["k"], x["v"], w.scale, w.causal, window=win)
        if w.backward:
            oracle.attn_bwd_ref(x["q"], x["k"], x["v"], x["do"], w.scale, w.causal, window=win)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    value = per_head * args.steps / el / 1e12
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        cores = len(os.sched_getaffinity(0))
    sample = (f"each step: 1 of {w.B * w.H} (batch, head) slices of {w.name} "
              f"({'fwd+bwd' if w.backward else 'fwd'}), fp64 NumPy oracle")
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(el * 1e3 / args.steps, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                      "causal": w.causal, "step": "oracle fwd+bwd" if w.backward else "oracle fwd"},
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=WORKLOAD_ORDER, default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--json-out", default=None)
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
