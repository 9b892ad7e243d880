#!/usr/bin/env python
"""Throughput of the MoE dispatch/combine hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole path over one batch of the 4096-token
prefill workload (hidden 7168, 256 experts in 8 logical ranks, top-8,
group-limited routing): dispatch layout, bf16 dispatch, FP8 dispatch, and
the gate-weighted combine of the bf16 receive buffer (identity experts).
Inputs are resident in HBM when the timed region starts.  Between steps the
L2 is flushed outside the per-step CUDA events: a 256 MiB write evicts the
step's data, then a 256 MiB read pushes the flush's own dirty lines back to
HBM, so no step pays for write-backs that are not its own.

Prints one JSON line.  ``value`` is algorithmic HBM bytes moved per second
over all ranks (each source byte read once, each destination byte written
once), the steps timed with events at their ends only; ``kernels`` and
``instrumented_step`` come from the same steps with events around every
kernel; ``roofline`` is the combine (the longest kernel) against the
measured copy bandwidth, timed live in the timed steps; ``decode`` is the
128-token decode workload in microseconds per call (layout + FP8 dispatch +
combine), unfused and with the fused layout + dispatch kernel, warm in
CUDA graphs of 20 calls and after an L2 flush; ``rank_dedup``,
``combine_variants`` (aligned layout, FP8 combine, expert replicas) and
``sm_budget_overlap`` (copy kernels beside a GEMM, with and without a
green-context SM partition) measure the further forms of the path;
``cpu_baseline`` times the CPU oracle on whole steps of the same batch;
``e2e`` runs the same step from pinned host buffers with the copies inside
the timed region; ``summary`` repeats the headline figures at the end.

Under torchrun (N > 1) every rank runs its own batch (weak scaling, no
data-path collective); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import re
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = ("dispatch+combine HBM GB/s (% of B200 peak); "
          "µs/call at 128-token decode")
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Write a buffer larger than L2 (evicting everything), then read another
    one so that the write's dirty lines are written back now rather than
    during the next timed kernel."""

    def __init__(self, device):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


# ------------------------------------------------------------- bytes model

def step_bytes(T: int, H: int, k: int, E: int, R: int) -> dict:
    """Algorithmic bytes per kernel of one step: each source byte read once,
    each destination byte written once (index arrays counted for layout
    only)."""
    N = T * k
    layout = T * k * 8 + (2 * E + 1 + 2 * R + 1) * 4 + T * R + 2 * N * 4
    return {
        "layout": layout,
        "dispatch_bf16": T * H * 2 + N * H * 2,
        "dispatch_fp8": T * H * 2 + N * H + N * (H // 128) * 4,
        "combine": N * H * 2 + T * H * 2,
    }


def decode_bytes(T, H, k, E, R) -> int:
    b = step_bytes(T, H, k, E, R)
    return b["layout"] + b["dispatch_fp8"] + b["combine"]


# --------------------------------------------------------------- utilities

def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every
    2 ms in a background thread while the timed region runs (plus one sample
    as it starts and one as it ends).  Read-only:
    no clock or other GPU setting is touched."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device):
        self.device = device
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.error = None
        self._stop = None
        self._thread = None

    def _handle(self, nv):
        props = torch.cuda.get_device_properties(self.device)
        try:
            return nv.nvmlDeviceGetHandleByUUID(("GPU-" + str(props.uuid)).encode())
        except Exception:  # noqa: BLE001 - fall back to the PCI address
            bus = (f"{getattr(props, 'pci_domain_id', 0):08x}:{props.pci_bus_id:02x}:"
                   f"{props.pci_device_id:02x}.0")
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - no NVML: report no clocks
            self.error = repr(e)
            return self
        self._stop = threading.Event()

        def sample():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, attr in self.REASONS:
                    if mask & getattr(nv, attr):
                        self.reasons.add(name)
                return True
            except Exception as e:  # noqa: BLE001
                self.error = repr(e)
                return False

        def run():
            while not self._stop.is_set() and sample():
                self._stop.wait(0.002)
            sample()

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "error": self.error}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of rank `rank`'s batch: every rank draws its own independent
    batch of the workload (weak scaling: the work per GPU is fixed)."""
    return rank


def job_value(bytes_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job GB/s: the bytes all ranks moved over the slowest rank's
    time."""
    return world * bytes_per_rank_step * steps / (max_ms * 1e-3) / 1e9


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------- the timed path

class Step:
    """Device buffers and the calls of one step on one GPU."""

    def __init__(self, ep, cfg, batch, device):
        self.ep, self.cfg, self.dev = ep, cfg, device
        T, H, k, E, R = batch.T, batch.H, cfg.k, cfg.E, cfg.R
        self.T, self.H = T, H
        self.idx = batch.idx.to(device)
        self.x = batch.x.to(device)
        self.w = batch.w.to(device)
        self.layout = ep.empty_layout(T, k, E, R, device)
        nws = ep.ep_layout_workspace_bytes(T, k, E, R)
        self.ws = torch.zeros(max(nws, 16), dtype=torch.uint8, device=device)
        self.d_err = torch.zeros(1, dtype=torch.int32, device=device)
        self.recv = torch.empty((T * k, H), dtype=torch.bfloat16, device=device)
        self.recv_q = torch.empty((T * k, H), dtype=torch.float8_e4m3fn, device=device)
        self.recv_s = torch.empty((T * k, H // 128), dtype=torch.float32, device=device)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=device)

    def run(self, stream, events=None, fp8_only=False, before_combine=None):
        ep, c = self.ep, self.cfg
        if events is not None:
            events[0].record(stream)
        ep.ep_get_layout(self.idx, c.E, c.R, out=self.layout, ws=self.ws,
                         d_err=self.d_err, stream=stream)
        if events is not None:
            events[1].record(stream)
        if not fp8_only:
            ep.ep_dispatch(self.x, self.layout.slot_pos, recv=self.recv,
                           d_err=self.d_err, stream=stream)
        if events is not None:
            events[2].record(stream)
        ep.ep_dispatch(self.x, self.layout.slot_pos, fp8=True, recv=self.recv_q,
                       recv_scale=self.recv_s, d_err=self.d_err, stream=stream)
        if events is not None:
            events[3].record(stream)
        if before_combine is not None:
            before_combine.record(stream)
        ep.ep_combine(self.recv, self.layout.slot_pos, self.w, out=self.out,
                      d_err=self.d_err, stream=stream)
        if events is not None:
            events[4].record(stream)


KERNELS = ("layout", "dispatch_bf16", "dispatch_fp8", "combine")


def workload_config(cfg, world: int) -> dict:
    """The `config` object of both arms: the prefill workload and the step."""
    return {
        "workload": ("prefill: T=4096 tokens, H=7168, E=256 experts in R=8 logical ranks, "
                     "top-8 group-limited routing; step = layout + bf16 dispatch + FP8 "
                     "dispatch + combine"),
        "T": cfg.T, "H": cfg.H, "E": cfg.E, "R": cfg.R, "k": cfg.k,
        "bytes_per_step": sum(step_bytes(cfg.T, cfg.H, cfg.k, cfg.E, cfg.R).values()),
        "l2": "flushed between steps outside the step events: 256 MiB write, then 256 MiB read",
        "parallelism": f"{world} independent batch(es), one per GPU",
    }


def bench_ours(args, world, rank, device):
    import combine_ep_get_09_b200 as ep
    ep.lib()
    cfg = workloads.CONFIGS["prefill"]
    batch = workloads.make_batch(cfg, seed=rank_seed(rank))
    st = Step(ep, cfg, batch, device)
    stream = torch.cuda.Stream(device)
    flush = L2Flush(device)
    nbytes = step_bytes(cfg.T, cfg.H, cfg.k, cfg.E, cfg.R)
    total_bytes = sum(nbytes.values())

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush()
            st.run(stream)
    stream.synchronize()
    if ep.ep_read_error(st.d_err, stream) != 0:
        raise RuntimeError("the device reported an error during warm-up")

    # timed region: K steps, each after the L2 flush, with CUDA events at
    # each step's start and end and one more right before the combine (the
    # dominant kernel, timed live for the roofline).  No other event sits
    # between kernels: one would make the next kernel wait for it and
    # cancel the programmatic launch overlap the kernels have when a caller
    # issues them back to back.
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(device)
    launches0 = ep.ep_kernel_launches()
    with ClockSampler(device) as clocks, torch.cuda.stream(stream):
        for a, c, b in evs:
            flush()
            a.record(stream)
            st.run(stream, before_combine=c)
            b.record(stream)
        stream.synchronize()
    torch.cuda.synchronize(device)
    barrier(world)
    launches = ep.ep_kernel_launches() - launches0
    if ep.ep_read_error(st.d_err, stream) != 0:
        raise RuntimeError("the device reported an error in the timed steps")
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, _, b in evs), world, device)
    combine_live_ms = max_over_ranks(statistics.mean(c.elapsed_time(b) for _, c, b in evs),
                                     world, device)
    instrumented = bench_instrumented(st, stream, flush, args.steps, world, device, nbytes)
    kern_ms = instrumented.pop("kernel_ms")
    peak, peak_kind = measured_peak()
    kernels = {}
    for n in KERNELS:
        gbs = nbytes[n] / (kern_ms[n] * 1e-3) / 1e9
        kernels[n] = {"us": round(kern_ms[n] * 1e3, 2), "bytes": nbytes[n],
                      "GB/s": round(gbs, 1), "frac_of_measured": round(gbs / peak, 4),
                      "frac_of_8TBs": round(gbs / SPEC_HBM_GBS, 4)}
    # the roofline kernel: the combine, the step's longest (checked against
    # the instrumented pass), timed live in the timed steps
    dom = "combine"
    longest = max(("dispatch_bf16", "dispatch_fp8", "combine"), key=lambda n: kern_ms[n])
    dom_gbs = nbytes[dom] / (combine_live_ms * 1e-3) / 1e9
    traffic = profiled_traffic(dom)

    value = job_value(total_bytes, args.steps, world, total_ms)
    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(cfg, world),
        "frac_of_8TBs": round(value / world / SPEC_HBM_GBS, 4),
        "kernels": kernels,
        "roofline": {"bound": "hbm", "kernel": dom, "longest_in_step": longest,
                     "us": round(combine_live_ms * 1e3, 2),
                     "achieved": round(dom_gbs, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(dom_gbs / peak, 4),
                     "traffic": traffic,
                     "algorithmic_bytes": nbytes[dom]},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "instrumented_step": instrumented,
    }
    if not args.skip_decode:
        result["decode"] = bench_decode(ep, device, world)
    if not args.skip_dedup:
        result["rank_dedup"] = bench_rank_dedup(ep, st, cfg, device, world)
    if not args.skip_workloads:
        result["other_workloads"] = bench_workloads(ep, device, world)
    if not args.skip_variants:
        result["combine_variants"] = bench_combine_variants(ep, st, cfg, device, world)
        result["combine_variants"]["replicas"] = bench_replicas(ep, device, world)
    if not args.skip_overlap:
        result["sm_budget_overlap"] = bench_overlap(ep, st, cfg, device, world)
    if not args.skip_e2e:
        result["e2e"] = bench_e2e(ep, cfg, batch, device, args, world, total_bytes)
    if world == 1 and rank == 0 and not args.skip_cpu:
        result["cpu_baseline"] = cpu_baseline(cfg, batch, args.cpu_seconds)
    # the headline figures once more, compactly, at the end of the line
    summary = {"step_GB/s": result["value"], "step_frac_of_8TBs": result["frac_of_8TBs"],
               "instrumented_step_GB/s": instrumented["step_GB/s"],
               "kernel_us": {n: kernels[n]["us"] for n in KERNELS},
               "kernel_frac_of_8TBs": {n: kernels[n]["frac_of_8TBs"] for n in KERNELS[1:]}}
    if "decode" in result:
        d = result["decode"]
        warm = next(v for k_, v in d.items() if k_.startswith("us_warm"))
        summary["decode_us_per_call"] = {
            "fused_warm_graph": warm["fused_call"], "unfused_warm_graph": warm["unfused_call"],
            "fused_cold_l2": d["us_cold_l2"]["fused_call"],
            "unfused_cold_l2": d["us_cold_l2"]["unfused_call"]}
    result["summary"] = summary
    return result


# Library sources each kernel is built from: a profile's DRAM traffic is
# only reported while these files are byte-for-byte the ones profiled.
KERNEL_SOURCES = {
    "layout": ("layout.cu", "ep_device.cuh"),
    "dispatch_bf16": ("dispatch_bf16.cu", "ep_device.cuh"),
    "dispatch_fp8": ("dispatch_fp8.cu", "fp8.cuh", "bulk.cuh", "ep_device.cuh"),
    "combine": ("combine.cu", "bulk.cuh", "ep_device.cuh"),
    "layout_dispatch_fp8": ("layout_dispatch.cu", "fp8.cuh", "bulk.cuh", "ep_device.cuh"),
    "combine_fp8": ("combine.cu", "bulk.cuh", "ep_device.cuh"),
}


def _code_only(text: str) -> str:
    """C/C++ source without its comments and blank lines (comments do not
    change a compiled kernel)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(l.rstrip() for l in text.splitlines() if l.strip())


def kernel_source_digest(kernel: str) -> str:
    """sha256 over the code (comments stripped) of the files a kernel's
    device code is built from, plus the #define constants of the public
    header."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "combine_ep_get_09_b200", "csrc", name)) as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    with open(os.path.join(ROOT, "include", "ep.h")) as f:
        h.update("".join(l for l in f if l.startswith("#define")).encode())
    return h.hexdigest()


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def profiled_traffic(kernel: str):
    """DRAM bytes per launch (read + write, one Nsight Compute capture of the
    prefill workload) recorded for `kernel` in profiles/traffic.json, or
    None when there is none or the kernel's sources changed since the
    capture (its recorded source_sha256 differs from the current one)."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha256") != kernel_source_digest(kernel):
        return None
    return float(rec["traffic_bytes_per_launch"])


def bench_rank_dedup(ep, st, cfg, device, world, iters=20):
    """The rank-deduplicated path on the same prefill batch: rank rows from
    the token-in-rank mask, dispatch into one row per (token, rank), and the
    unit-weight combine of per-rank partial outputs.  Each kernel is timed
    alone (flushed L2) and reported with its algorithmic bytes."""
    T, H, R = cfg.T, cfg.H, cfg.R
    stream = torch.cuda.Stream(device)
    flush = L2Flush(device)
    with torch.cuda.stream(stream):
        st.run(stream)
        rl = ep.ep_get_rank_layout(st.layout.in_rank, stream=stream)
    stream.synchronize()
    rows = int(rl.off_r[-1].item())
    recv = torch.empty((T * R, H), dtype=torch.bfloat16, device=device)
    q = torch.empty((T * R, H), dtype=torch.float8_e4m3fn, device=device)
    sc = torch.empty((T * R, H // 128), dtype=torch.float32, device=device)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    calls = {
        "rank_layout": (lambda: ep.ep_get_rank_layout(st.layout.in_rank, out=rl, stream=stream),
                        T * R + (2 * R + 1) * 4 + 2 * T * R * 4),
        "dispatch_bf16": (lambda: ep.ep_dispatch(st.x, rl.rank_row, recv=recv, stream=stream),
                          T * H * 2 + rows * H * 2),
        "dispatch_fp8": (lambda: ep.ep_dispatch(st.x, rl.rank_row, fp8=True, recv=q,
                                                recv_scale=sc, stream=stream),
                         T * H * 2 + rows * (H + H // 32)),
        "combine": (lambda: ep.ep_combine(recv, rl.rank_row, None, out=out, stream=stream),
                    rows * H * 2 + T * H * 2),
    }
    res = {"rows": rows, "expert_rows": T * cfg.k,
           "write_saving": round(1 - rows / (T * cfg.k), 4)}
    for name, (fn, nbytes) in calls.items():
        evs = []
        with torch.cuda.stream(stream):
            for _ in range(3):
                flush()
                fn()
            for _ in range(iters):
                flush()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                evs.append((a, b))
        stream.synchronize()
        us = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3,
                            world, device)
        res[name] = {"us": round(us, 2), "bytes": nbytes,
                     "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1)}
    return res


def bench_instrumented(st, stream, flush, steps, world, device, nbytes):
    """The same steps once more, after the timed region, with CUDA events
    around every kernel: each kernel's device time inside the step (it
    starts after the previous kernel's completion, as the events force, so
    the sum exceeds the step timed without them)."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        for e in evs:
            flush()
            st.run(stream, e)
        stream.synchronize()
    barrier(world)
    per_kernel = {n: [] for n in KERNELS}
    for e in evs:
        for j, n in enumerate(KERNELS):
            per_kernel[n].append(e[j].elapsed_time(e[j + 1]))
    ms = max_over_ranks(sum(e[0].elapsed_time(e[4]) for e in evs), world, device)
    total_bytes = sum(nbytes.values())
    return {"kernel_ms": {n: max_over_ranks(statistics.mean(v), world, device)
                          for n, v in per_kernel.items()},
            "step_GB/s": round(job_value(total_bytes, steps, world, ms), 1),
            "us_per_step": round(ms / steps * 1e3, 2), "steps": steps,
            "how": "events around every kernel of each step; the same L2 flush between steps"}


def bench_workloads(ep, device, world, names=("skewed", "large"), iters=10):
    """The step's kernels on the other full-size shapes, each step after an
    L2 flush, timed with CUDA events around each kernel (like the prefill
    step): the skewed batch (Zipf-popular experts, 8192 tokens) and the large
    one (32768 tokens of H=4096 over 128 experts in 16 ranks)."""
    res = {}
    for name in names:
        cfg = workloads.CONFIGS[name]
        st = Step(ep, cfg, workloads.make_batch(cfg, seed=0), device)
        stream = torch.cuda.Stream(device)
        flush = L2Flush(device)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(iters)]
        with torch.cuda.stream(stream):
            for _ in range(3):
                flush()
                st.run(stream)
            for e in evs:
                flush()
                st.run(stream, e)
        stream.synchronize()
        if ep.ep_read_error(st.d_err, stream) != 0:
            raise RuntimeError(f"the device reported an error on the {name} workload")
        nbytes = step_bytes(cfg.T, cfg.H, cfg.k, cfg.E, cfg.R)
        out = {"T": cfg.T, "H": cfg.H, "E": cfg.E, "R": cfg.R, "k": cfg.k}
        for j, n in enumerate(KERNELS):
            us = max_over_ranks(statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) * 1e3,
                                world, device)
            gbs = nbytes[n] / (us * 1e-6) / 1e9
            out[n] = {"us": round(us, 2), "bytes": nbytes[n], "GB/s": round(gbs, 1),
                      "frac_of_8TBs": round(gbs / SPEC_HBM_GBS, 4)}
        step_us = max_over_ranks(statistics.mean(e[0].elapsed_time(e[4]) for e in evs) * 1e3,
                                 world, device)
        out["step_us"] = round(step_us, 2)
        out["step_GB/s"] = round(sum(nbytes.values()) / (step_us * 1e-6) / 1e9, 1)
        res[name] = out
        del st
        torch.cuda.empty_cache()
    return res


def bench_combine_variants(ep, st, cfg, device, world, iters=20, align=128):
    """The combine variants on the prefill batch, each kernel timed alone
    (flushed L2): the aligned layout for a grouped GEMM with `align`-row
    tiles, the FP8 dispatch into that padded buffer, and the combine of FP8
    expert outputs (the FP8 receive rows themselves: identity experts)."""
    T, H, k, E = cfg.T, cfg.H, cfg.k, cfg.E
    stream = torch.cuda.Stream(device)
    flush = L2Flush(device)
    with torch.cuda.stream(stream):
        st.run(stream)
        pl = ep.ep_pad_layout(st.layout, align, stream=stream)
    stream.synchronize()
    cap = ep.ep_aligned_rows(T, k, E, align)
    q = torch.zeros((cap, H), dtype=torch.float8_e4m3fn, device=device)
    sc = torch.zeros((cap, H // 128), dtype=torch.float32, device=device)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    N = T * k
    calls = {
        "pad_layout": (lambda: ep.ep_pad_layout(st.layout, align, out=pl, stream=stream),
                       E * 4 + N * 4 + (E + 1) * 4 + N * 4 + cap * 4),
        "dispatch_fp8_padded": (lambda: ep.ep_dispatch(st.x, pl.slot_pos, fp8=True, recv=q,
                                                       recv_scale=sc, d_err=st.d_err,
                                                       stream=stream),
                                T * H * 2 + N * (H + H // 32)),
        "combine_fp8": (lambda: ep.ep_combine_fp8(q, sc, pl.slot_pos, st.w, out=out,
                                                  d_err=st.d_err, stream=stream),
                        N * (H + H // 32) + T * H * 2),
    }
    res = {"align": align, "rows": cap, "rows_in_use": None}
    for name, (fn, nbytes) in calls.items():
        evs = []
        with torch.cuda.stream(stream):
            for _ in range(3):
                flush()
                fn()
            for _ in range(iters):
                flush()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                evs.append((a, b))
        stream.synchronize()
        us = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3,
                            world, device)
        res[name] = {"us": round(us, 2), "bytes": nbytes,
                     "GB/s": round(nbytes / (us * 1e-6) / 1e9, 1)}
    res["rows_in_use"] = int(pl.off_pad[-1].item())
    if ep.ep_read_error(st.d_err, stream) != 0:
        raise RuntimeError("the device reported an error in the combine variants")
    return res


def bench_replicas(ep, device, world, iters=20, hot=16, copies=4):
    """Redundant copies of the busiest experts on the skewed batch: the
    `hot` most loaded of 256 experts get `copies` copies each (304 physical
    experts in 8 ranks).  Times the replica mapping kernel and the layout of
    the physical ids (each alone, flushed L2) and reports the busiest
    expert's load before and after."""
    cfg = workloads.CONFIGS["skewed"]
    batch = workloads.make_batch(cfg, seed=300, H=8)
    E, R, T, k = cfg.E, cfg.R, cfg.T, cfg.k
    idx = batch.idx.to(device)
    load = np.bincount(batch.idx.numpy().reshape(-1), minlength=E)
    n_rep = np.ones(E, np.int64)
    n_rep[np.argsort(-load, kind="stable")[:hot]] = copies
    rep_off = torch.from_numpy(np.concatenate([[0], np.cumsum(n_rep)]).astype(np.int32)).to(device)
    E_phys = int(n_rep.sum())
    rep_ids = torch.arange(E_phys, dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device)
    flush = L2Flush(device)
    d_err = torch.zeros(1, dtype=torch.int32, device=device)
    with torch.cuda.stream(stream):
        L = ep.ep_get_layout(idx, E, R, d_err=d_err, stream=stream)
        phys = ep.ep_map_replicas(idx, L, rep_off, rep_ids, d_err=d_err, stream=stream)
        P = ep.ep_get_layout(phys, E_phys, R, d_err=d_err, stream=stream)
    stream.synchronize()
    N = T * k
    calls = {"map_replicas": (lambda: ep.ep_map_replicas(idx, L, rep_off, rep_ids, out=phys,
                                                         d_err=d_err, stream=stream),
                              N * (8 + 4 + 4)),
             "physical_layout": (lambda: ep.ep_get_layout(phys, E_phys, R, out=P, d_err=d_err,
                                                          stream=stream),
                                 N * 4 + N * 8 + T * R)}
    res = {"workload": f"skewed: T={T}, E={E} in R={R}, top-{k}; the {hot} busiest experts "
                       f"get {copies} copies ({E_phys} physical experts)",
           "max_load_logical": int(load.max()), "mean_load": round(float(load.mean()), 1),
           "max_load_physical": int(P.cnt_e.max().item())}
    for name, (fn, nbytes) in calls.items():
        evs = []
        with torch.cuda.stream(stream):
            for _ in range(3):
                flush()
                fn()
            for _ in range(iters):
                flush()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                evs.append((a, b))
        stream.synchronize()
        us = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3,
                            world, device)
        res[name] = {"us": round(us, 2), "bytes": nbytes}
    if ep.ep_read_error(d_err, stream) != 0:
        raise RuntimeError("the device reported an error in the replica runs")
    return res


OVERLAP_GEMM = (4096, 7168, 2048)   # M, K, N of the stand-in expert GEMM
OVERLAP_SMS = (16, 32, 64, 148)
GREEN_SMS = (16, 32, 48)


class GreenPartition:
    """Two disjoint SM partitions of the device through CUDA green contexts:
    about `n_comm` SMs for the copy kernels, the rest for the GEMM, each
    with its own stream.  Work launched into a partition's stream runs on
    that partition's SMs only.  Read-only towards the device's settings:
    nothing outlives the process (close() releases everything)."""

    def __init__(self, device, n_comm):
        from cuda.bindings import driver as drv
        self.drv = drv
        self.ok(drv.cuInit(0))
        dev, = self.ok(drv.cuDeviceGet(torch.device(device).index or 0))
        res, = self.ok(drv.cuDeviceGetDevResource(
            dev, drv.CUdevResourceType.CU_DEV_RESOURCE_TYPE_SM))
        groups, _, rest = self.ok(drv.cuDevSmResourceSplitByCount(1, res, 0, n_comm))
        self.n_comm = int(groups[0].sm.smCount)
        self.n_rest = int(rest.sm.smCount)
        flag = drv.CUgreenCtxCreate_flags.CU_GREEN_CTX_DEFAULT_STREAM
        nb = drv.CUstream_flags.CU_STREAM_NON_BLOCKING
        self.ctxs, self.streams, self.events = [], [], []
        for r in (groups[0], rest):
            desc, = self.ok(drv.cuDevResourceGenerateDesc([r], 1))
            g, = self.ok(drv.cuGreenCtxCreate(desc, dev, flag))
            self.ctxs.append(g)
            st, = self.ok(drv.cuGreenCtxStreamCreate(g, nb, 0))
            self.streams.append(st)
            # an event of the partition's own context marks the end of its work
            ctx, = self.ok(drv.cuCtxFromGreenCtx(g))
            self.ok(drv.cuCtxPushCurrent(ctx))
            ev, = self.ok(drv.cuEventCreate(drv.CUevent_flags.CU_EVENT_DISABLE_TIMING))
            self.ok(drv.cuCtxPopCurrent())
            self.events.append(ev)
        self.comm = torch.cuda.ExternalStream(int(self.streams[0]), device=device)
        self.comp = torch.cuda.ExternalStream(int(self.streams[1]), device=device)

    def ok(self, r):
        err = r[0] if isinstance(r, tuple) else r
        if err != self.drv.CUresult.CUDA_SUCCESS:
            raise RuntimeError(f"green context: {err}")
        return r[1:] if isinstance(r, tuple) else ()

    def timed(self, device, comm, comp):
        """Device microseconds from a start event on a plain stream, which
        both partitions wait on, until both partitions' work is done."""
        drv = self.drv
        s0 = torch.cuda.current_stream(device)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s0)
        for st in self.streams:
            self.ok(drv.cuStreamWaitEvent(st, drv.CUevent(a.cuda_event), 0))
        if comm is not None:
            with torch.cuda.stream(self.comm):
                comm()
        if comp is not None:
            with torch.cuda.stream(self.comp):
                comp()
        for st, ev in zip(self.streams, self.events):
            self.ok(drv.cuEventRecord(ev, st))
            self.ok(drv.cuStreamWaitEvent(drv.CUstream(s0.cuda_stream), ev, 0))
        b.record(s0)
        torch.cuda.synchronize(device)
        return a.elapsed_time(b) * 1e3

    def close(self):
        drv = self.drv
        torch.cuda.synchronize()
        for st in self.streams:
            drv.cuStreamDestroy(st)
        for ev in self.events:
            drv.cuEventDestroy(ev)
        for g in self.ctxs:
            drv.cuGreenCtxDestroy(g)


def bench_green_overlap(ep, st, device, world, ops, gemm, flush, gemm_full_us, reps=10):
    """The copy kernels confined to an SM partition beside the GEMM on the
    other partition (green contexts), against both on all SMs one after the
    other."""
    res = {"baseline": "both on all 148 SMs, one after the other", "rows": []}
    for S in GREEN_SMS:
        part = GreenPartition(device, S)
        try:
            def med(fn):
                fn()
                vals = []
                for _ in range(reps):
                    torch.cuda.synchronize(device)
                    flush()
                    torch.cuda.synchronize(device)
                    vals.append(fn())
                return statistics.median(vals)
            gemm_rest = med(lambda: part.timed(device, None, gemm))
            row = {"comm_sms": part.n_comm, "gemm_sms": part.n_rest,
                   "gemm_alone_us": round(max_over_ranks(gemm_rest, world, device), 2)}
            for name, (op, full_us) in ops.items():
                alone = med(lambda: part.timed(device, lambda: op(part.n_comm), None))
                both = med(lambda: part.timed(device, lambda: op(part.n_comm), gemm))
                alone = max_over_ranks(alone, world, device)
                both = max_over_ranks(both, world, device)
                row[name] = {"alone_us": round(alone, 2), "both_us": round(both, 2),
                             "serial_all_sms_us": round(full_us + gemm_full_us, 2),
                             "speedup": round((full_us + gemm_full_us) / both, 3)}
            res["rows"].append(row)
        finally:
            part.close()
    return res


def bench_overlap(ep, st, cfg, device, world, reps=10):
    """SM-budgeted dispatch and combine beside a GEMM on another stream.

    DeepEP's normal kernels run on a fixed budget of SMs so that the rest
    can compute at the same time (frogred8 blog, "deepEP optimization",
    third method: the SM count is a parameter).  The GEMM stands in for the
    expert computation (cuBLAS through torch.matmul, bf16, M x K @ K x N).
    For each SM budget S: the bf16 dispatch (or combine) alone with
    num_sms=S, the GEMM alone, and both launched together on two streams;
    `both_us` runs from a common start event until both streams are done
    (L2 flushed before each trial).  `overlap` = (alone + gemm) / both:
    1 means no overlap, 2 perfect overlap of equal halves."""
    M, K, N = OVERLAP_GEMM
    gen = torch.Generator(device=device).manual_seed(7)
    A = torch.randn((M, K), device=device, dtype=torch.bfloat16, generator=gen)
    B = torch.randn((K, N), device=device, dtype=torch.bfloat16, generator=gen)
    Cm = torch.empty((M, N), device=device, dtype=torch.bfloat16)
    s_comm = torch.cuda.Stream(device)
    s_comp = torch.cuda.Stream(device)
    flush = L2Flush(device)
    with torch.cuda.stream(s_comm):
        st.run(s_comm)   # a valid layout and receive buffer
    s_comm.synchronize()

    def gemm():
        torch.matmul(A, B, out=Cm)

    ops = {
        "dispatch_bf16": lambda S, s=None: ep.ep_dispatch(
            st.x, st.layout.slot_pos, recv=st.recv, num_sms=S, d_err=st.d_err,
            stream=s_comm if s is None else s),
        "combine": lambda S, s=None: ep.ep_combine(
            st.recv, st.layout.slot_pos, st.w, out=st.out, num_sms=S, d_err=st.d_err,
            stream=s_comm if s is None else s),
    }

    def op_on(op, S):
        # the current stream (the partition's, inside GreenPartition.timed)
        op(S, torch.cuda.current_stream(device))

    def trial(comm, comp):
        """Device microseconds from a common start until both streams end."""
        torch.cuda.synchronize(device)
        flush()
        torch.cuda.synchronize(device)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(s_comm)
        s_comp.wait_event(ev[0])
        if comm is not None:
            with torch.cuda.stream(s_comm):
                comm()
        if comp is not None:
            with torch.cuda.stream(s_comp):
                comp()
        ev[1].record(s_comm)
        ev[2].record(s_comp)
        torch.cuda.synchronize(device)
        return max(ev[0].elapsed_time(ev[1]), ev[0].elapsed_time(ev[2])) * 1e3

    def median(fn):
        fn()
        return statistics.median(fn() for _ in range(reps))

    gemm_us = median(lambda: trial(None, gemm))
    res = {"gemm": {"mkn": [M, K, N], "us": round(max_over_ranks(gemm_us, world, device), 2),
                    "TFLOP/s": round(2 * M * K * N / (gemm_us * 1e-6) / 1e12, 1)},
           "note": "both_us = dispatch or combine and the GEMM on two streams at once"}
    full = {}
    for name, op in ops.items():
        rows = []
        for S in OVERLAP_SMS:
            alone = median(lambda: trial(lambda: op(S), None))
            both = median(lambda: trial(lambda: op(S), gemm))
            alone = max_over_ranks(alone, world, device)
            both = max_over_ranks(both, world, device)
            rows.append({"num_sms": S, "alone_us": round(alone, 2), "both_us": round(both, 2),
                         "serial_us": round(alone + gemm_us, 2),
                         "overlap": round((alone + gemm_us) / both, 3)})
            if S == OVERLAP_SMS[-1]:
                full[name] = alone
        res[name] = rows
    # the same with the copy kernels confined to an SM partition (one GPU
    # only: a failure on one rank must not leave the others in a collective)
    if world == 1:
        try:
            comm_ops = {name: (lambda S, op=op: op_on(op, S), full[name])
                        for name, op in ops.items()}
            res["green_contexts"] = bench_green_overlap(ep, st, device, world, comm_ops, gemm,
                                                        flush, gemm_us)
        except Exception as e:  # noqa: BLE001 - reported, not fatal
            res["green_contexts"] = {"error": repr(e)[:300]}
    else:
        res["green_contexts"] = {"skipped": "measured with one GPU only"}
    if ep.ep_read_error(st.d_err, s_comm) != 0:
        raise RuntimeError("the device reported an error in the overlap runs")
    return res


def bench_decode(ep, device, world, calls=20, reps=10, cold_reps=10):
    """The 128-token decode workload: µs per call of layout + FP8 dispatch +
    combine, fused (ep_layout_dispatch + combine, two kernels) and unfused
    (three kernels), and of each kernel alone.

    warm: `calls` back-to-back calls captured in one CUDA graph and the
    graph replayed `reps` times (the form a decode step's graph has: the
    calls overlap their launch latency through programmatic dependent
    launch, and the graph's own launch is paid once per `calls` calls); the
    working set stays in L2.  cold: `cold_reps` pairs of (L2 flush, call) in
    one graph, less the same graph without the calls, per call (single
    calls timed with their own events read in steps of about 1-2 us on this
    part)."""
    cfg = workloads.CONFIGS["decode"]
    batch = workloads.make_batch(cfg, seed=100)
    st = Step(ep, cfg, batch, device)
    stream = torch.cuda.Stream(device)
    flush = L2Flush(device)
    c = cfg

    def layout():
        ep.ep_get_layout(st.idx, c.E, c.R, out=st.layout, ws=st.ws, d_err=st.d_err,
                         stream=stream)

    def dispatch_fp8():
        ep.ep_dispatch(st.x, st.layout.slot_pos, fp8=True, recv=st.recv_q,
                       recv_scale=st.recv_s, d_err=st.d_err, stream=stream)

    def layout_dispatch():
        ep.ep_layout_dispatch(st.idx, c.E, c.R, st.x, True, out=st.layout, recv=st.recv_q,
                              recv_scale=st.recv_s, ws=st.ws, d_err=st.d_err, stream=stream)

    def combine():
        ep.ep_combine(st.recv, st.layout.slot_pos, st.w, out=st.out, d_err=st.d_err,
                      stream=stream)

    def unfused():
        layout()
        dispatch_fp8()
        combine()

    def fused():
        layout_dispatch()
        combine()

    with torch.cuda.stream(stream):
        for _ in range(20):
            st.run(stream, fp8_only=True)
            fused()
    stream.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def warm_us(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(calls):
                fn()
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
            a.record(stream)
            for _ in range(reps):
                g.replay()
            b.record(stream)
        stream.synchronize()
        del g
        return a.elapsed_time(b) * 1e3 / (reps * calls)

    def graph_total_us(body):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            body()
        with torch.cuda.stream(stream):
            g.replay()
            a.record(stream)
            for _ in range(reps):
                g.replay()
            b.record(stream)
        stream.synchronize()
        del g
        return a.elapsed_time(b) * 1e3 / reps

    def flushes():
        for _ in range(cold_reps):
            flush()

    flush_us = graph_total_us(flushes)

    def cold_us(fn):
        def body():
            for _ in range(cold_reps):
                flush()
                fn()
        return (graph_total_us(body) - flush_us) / cold_reps

    fns = {"fused_call": fused, "unfused_call": unfused, "layout": layout,
           "dispatch_fp8": dispatch_fp8, "layout_dispatch_fp8": layout_dispatch,
           "combine": combine}
    warm = {n: round(max_over_ranks(warm_us(f), world, device), 2) for n, f in fns.items()}
    cold = {n: round(max_over_ranks(cold_us(f), world, device), 2) for n, f in fns.items()}
    if ep.ep_read_error(st.d_err, stream) != 0:
        raise RuntimeError("the device reported an error in the decode calls")
    nb = decode_bytes(cfg.T, cfg.H, cfg.k, cfg.E, cfg.R)
    return {"workload": "decode: T=128, H=7168, E=256/R=8, top-8, FP8 dispatch; "
                        "call = layout + FP8 dispatch + combine",
            "fused": "ep_layout_dispatch (layout + FP8 dispatch, one kernel) + ep_combine",
            "unfused": "ep_get_layout + ep_dispatch(fp8) + ep_combine",
            "us_warm_graph_of_%d" % calls: warm,
            "us_cold_l2": cold,
            "bytes_per_call": nb,
            "GB/s_warm_fused": round(nb / (warm["fused_call"] * 1e-6) / 1e9, 1),
            "how": (f"warm: {calls} back-to-back calls (or kernel launches) in one CUDA graph, "
                    f"replayed {reps} times; cold: {cold_reps} (L2 flush, call) pairs in one "
                    "graph less the flushes alone, per call"),
            "pages_context_us": 163.0}


def bench_e2e(ep, cfg, batch, device, args, world, total_bytes):
    """Same step end to end from pinned host buffers: every step copies its
    inputs (idx, w, x) host->device and its combined output device->host.
    Steps are pipelined over three streams (copy-in, compute, copy-out) and
    two device buffer sets, so step i+1's upload and step i-1's download
    overlap step i's kernels; the time is from the first upload's start to
    the last download's end, on the device."""
    T, H = cfg.T, cfg.H
    h_idx = batch.idx.pin_memory()
    h_w = batch.w.pin_memory()
    h_x = batch.x.pin_memory()
    h_out = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    sets = [Step(ep, cfg, batch, device) for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))

    def run(n, first_ev=None, last_ev=None):
        comp_done = [None, None]
        out_done = [None, None]
        for i in range(n):
            b = i % 2
            st = sets[b]
            with torch.cuda.stream(s_in):
                if comp_done[b] is not None:
                    s_in.wait_event(comp_done[b])      # buffer set free again
                if i == 0 and first_ev is not None:
                    first_ev.record(s_in)
                st.idx.copy_(h_idx, non_blocking=True)
                st.w.copy_(h_w, non_blocking=True)
                st.x.copy_(h_x, non_blocking=True)
                in_done = torch.cuda.Event()
                in_done.record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(in_done)
                if out_done[b] is not None:
                    s_comp.wait_event(out_done[b])     # output buffer downloaded
                st.run(s_comp)
                comp_done[b] = torch.cuda.Event()
                comp_done[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                h_out[b].copy_(st.out, non_blocking=True)
                out_done[b] = torch.cuda.Event()
                out_done[b].record(s_out)
        if last_ev is not None:
            last_ev.record(s_out)

    run(max(3, args.warmup))
    torch.cuda.synchronize(device)
    n = max(4, min(args.steps, 20))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    run(n, t0, t1)
    torch.cuda.synchronize(device)
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world, device)
    h2d = h_idx.numel() * 8 + h_w.numel() * 4 + h_x.numel() * 2
    d2h = h_out[0].numel() * 2
    return {"value": round(job_value(total_bytes, n, world, ms), 1), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms / n, 4), "steps": n,
            "how": "pinned host buffers, 3 streams (upload / kernels / download), "
                   "2 device buffer sets, steps overlapped"}


# ------------------------------------------------------------ CPU oracle

def oracle_sample_step(oracle, cfg, x, idx, w):
    """One pass of the oracle over a token sample: layout, bf16 dispatch,
    FP8 dispatch, combine (identity experts)."""
    T, k = idx.shape
    L = oracle.layout(idx, cfg.E, cfg.R)
    recv = oracle.dispatch_bf16(x, L["slot_pos"], T * k)
    oracle.dispatch_fp8(x, L["slot_pos"], T * k)
    oracle.combine(recv, L["slot_pos"], w)


def cpu_baseline(cfg, batch, seconds: float):
    """The oracle as it stands, single-threaded, on whole steps of the same
    prefill batch the GPU times (all T tokens), repeated for about
    `seconds`; then every host core at once (cpu_baseline_threads)."""
    import oracle
    x, idx, w = batch.x, batch.idx, batch.w
    nb = sum(step_bytes(batch.T, cfg.H, cfg.k, cfg.E, cfg.R).values())
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_sample_step(oracle, cfg, x, idx, w)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    res = {"value": round(nb * reps / el / 1e9, 3), "unit": "GB/s", "cores": 1,
           "kind": "oracle",
           "sample": (f"the whole {batch.T}-token prefill batch per step (layout + bf16 "
                      f"dispatch + FP8 dispatch + combine), {reps} steps in {el:.1f} s, "
                      "single-threaded C oracle")}
    res["all_cores"] = cpu_baseline_threads(cfg, batch, seconds, nb)
    return res


def cpu_baseline_threads(cfg, batch, seconds: float, nb: int, max_threads: int = 64):
    """The same oracle step on every host core at once: the batch's tokens
    split into one contiguous slice per core (one Python thread each; the C
    oracle runs without the interpreter lock), every thread repeating the
    step on its slice for about `seconds`.  The slices together are the
    whole batch, so the bytes of one pass over all of them equal one step's."""
    import threading
    import oracle
    n = max(1, min(len(os.sched_getaffinity(0)), max_threads, batch.T))
    bounds = [batch.T * i // n for i in range(n + 1)]
    slices = [tuple(t[bounds[i]:bounds[i + 1]].contiguous() for t in (batch.x, batch.idx, batch.w))
              for i in range(n)]
    reps = [0] * n
    start = threading.Barrier(n + 1)
    stop = time.perf_counter() + 1e9

    def work(i):
        x, idx, w = slices[i]
        start.wait()
        while time.perf_counter() < stop:
            oracle_sample_step(oracle, cfg, x, idx, w)
            reps[i] += 1

    threads = [threading.Thread(target=work, args=(i,), daemon=True) for i in range(n)]
    for t in threads:
        t.start()
    t0 = time.perf_counter()
    stop = t0 + seconds
    start.wait()
    for t in threads:
        t.join()
    el = time.perf_counter() - t0
    done = sum(reps[i] * (bounds[i + 1] - bounds[i]) for i in range(n)) / batch.T
    return {"value": round(nb * done / el / 1e9, 3), "unit": "GB/s", "cores": n,
            "kind": "oracle",
            "sample": (f"{n} threads, each repeating the step on its own 1/{n} of the "
                       f"{batch.T}-token prefill batch; {done:.1f} batches' worth in {el:.1f} s")}


def bench_reference(args, world, rank):
    """The oracle as it stands, timed on the host cores: same metric, unit
    and workload as the GPU arm -- every step is the whole 4096-token
    prefill batch (layout + bf16 dispatch + FP8 dispatch + combine),
    single-threaded."""
    if rank != 0:
        return None
    import oracle
    cfg = workloads.CONFIGS["prefill"]
    batch = workloads.make_batch(cfg, seed=0)
    x, idx, w = batch.x, batch.idx, batch.w
    nb = sum(step_bytes(cfg.T, cfg.H, cfg.k, cfg.E, cfg.R).values())
    for _ in range(args.warmup):
        oracle_sample_step(oracle, cfg, x, idx, w)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(oracle, cfg, x, idx, w)
    el = time.perf_counter() - t0
    value = nb * args.steps / el / 1e9
    sample = (f"the whole {cfg.T}-token prefill batch per step, {args.steps} steps after "
              f"{args.warmup} warm-up steps; single-threaded C oracle")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el * 1e3 / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(cfg, world),
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": 1,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def profile_kernel(args, device):
    """Runs one kernel of the path by itself (or, with --profile step, the
    whole step), --steps times after --warmup warm-ups, with the L2 flush
    before each launch: the small, repeatable command that Nsight Compute
    captures are taken on.  Prints the mean CUDA-event time of the call (not
    a benchmark line)."""
    import combine_ep_get_09_b200 as ep
    cfg = workloads.CONFIGS[args.workload]
    st = Step(ep, cfg, workloads.make_batch(cfg, seed=0), device)
    stream = torch.cuda.Stream(device)
    flush = L2Flush(device)
    c = cfg
    calls = {
        "layout": lambda: ep.ep_get_layout(st.idx, c.E, c.R, out=st.layout, ws=st.ws,
                                           d_err=st.d_err, stream=stream),
        "dispatch_bf16": lambda: ep.ep_dispatch(st.x, st.layout.slot_pos, recv=st.recv,
                                                d_err=st.d_err, stream=stream),
        "dispatch_fp8": lambda: ep.ep_dispatch(st.x, st.layout.slot_pos, fp8=True,
                                               recv=st.recv_q, recv_scale=st.recv_s,
                                               d_err=st.d_err, stream=stream),
        "combine": lambda: ep.ep_combine(st.recv, st.layout.slot_pos, st.w, out=st.out,
                                         d_err=st.d_err, stream=stream),
        "layout_dispatch_fp8": lambda: ep.ep_layout_dispatch(
            st.idx, c.E, c.R, st.x, True, out=st.layout, recv=st.recv_q,
            recv_scale=st.recv_s, ws=st.ws, d_err=st.d_err, stream=stream),
        "combine_fp8": lambda: ep.ep_combine_fp8(st.recv_q, st.recv_s, st.layout.slot_pos, st.w,
                                                 out=st.out, d_err=st.d_err, stream=stream),
    }
    # the whole step, for captures of a kernel in the state the previous
    # kernels of the step leave (with ncu --cache-control none)
    calls["step"] = lambda: st.run(stream)
    call = calls[args.profile]
    with torch.cuda.stream(stream):
        st.run(stream)
        for _ in range(args.warmup):
            flush()
            call()
        ts = []
        for _ in range(args.steps):
            flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            ts.append((a, b))
    stream.synchronize()
    if ep.ep_read_error(st.d_err, stream) != 0:
        raise RuntimeError("the device reported an error")
    us = statistics.mean(a.elapsed_time(b) for a, b in ts) * 1e3
    print(json.dumps({"profile": args.profile, "workload": args.workload,
                      "launches_timed": args.steps, "us_mean": round(us, 2)}))


def main():
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--skip-decode", action="store_true")
    p.add_argument("--skip-e2e", action="store_true")
    p.add_argument("--skip-cpu", action="store_true")
    p.add_argument("--skip-dedup", action="store_true")
    p.add_argument("--skip-overlap", action="store_true")
    p.add_argument("--skip-variants", action="store_true")
    p.add_argument("--skip-workloads", action="store_true",
                   help="skip the skewed and large shapes")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--profile", choices=("layout", "dispatch_bf16", "dispatch_fp8", "combine",
                                         "layout_dispatch_fp8", "combine_fp8", "step"),
                   help="run only this kernel (for profiler captures)")
    p.add_argument("--workload", choices=tuple(workloads.CONFIGS), default="prefill",
                   help="workload of --profile")
    args = p.parse_args()
    if args.warmup < 3:
        p.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)

    if args.impl == "reference":
        res = bench_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.profile:
        profile_kernel(args, device)
        return
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    try:
        res = bench_ours(args, world, rank, device)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
