#!/usr/bin/env python
"""Benchmark of the MonarchAttention forward pass on B200; prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one full forward call (every kernel of the path) over one batch of
synthetic inputs already resident in device memory.  Inputs rotate over
several copies whose total exceeds the 126 MB L2 several times, so every step
reads its Q/K/V from HBM.  Multi-GPU runs (torchrun, one rank per GPU) give
every rank its own batch (independent heads: weak scaling, no collective on
the data path) and report the max over ranks of the device time.

Keys beyond the base contract: "e2e" (the same metric through the host-buffer
C-ABI call, copies included), "roofline" (dominant kernel, CUDA events taken
live in this run), "cpu_baseline" (the float64 oracle on the host cores, on a
bounded sample), "clocks" (SM clock and throttle reasons sampled while the
timed calls run), "gpu_launches" (kernels launched in the timed region).
"""
from __future__ import annotations

import argparse
import datetime
import faulthandler
import hashlib
import json
import math
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from structured_sub_quadratic_b200.inputs import WORKLOADS, Workload, make_inputs  # noqa: E402

faulthandler.enable()


def log(msg):
    """Progress marker on stderr (stdout carries only the JSON line)."""
    print(f"[bench] {msg}", file=sys.stderr, flush=True)


METRIC = "MonarchAttention fwd ms/call & TFLOP/s at 1 B200; % tensor-pipe/HBM roofline"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# FP32 FFMA peak of the SIMT kernels: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz.
ALU_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# ---------------------------------------------------------------------------
# algorithmic work model
# ---------------------------------------------------------------------------
def alg_flops(wl: Workload) -> float:
    """2 N d [(2T+1) c1 b2 + 2T c2 b1] per head: T R-updates (logits + R K),
    Y = R V once, T L-updates (logits + aggregation or output)."""
    N, d, T = wl.N, wl.d, wl.T
    return wl.heads * 2.0 * N * d * ((2 * T + 1) * wl.c1 * wl.b2 + 2 * T * wl.c2 * wl.b1)


def elt_bytes(wl: Workload) -> int:
    return 4 if wl.dtype == torch.float32 else 2


def alg_bytes(wl: Workload) -> float:
    """Q, K, V read once and O written once: 4 N d elements per head."""
    return wl.heads * 4.0 * wl.N * wl.d * elt_bytes(wl)


def kernel_work(name: str, wl: Workload):
    """(FLOPs, bytes) of one launch of kernel `name` on wl, algorithmically.

    FLOPs: the kernel's share of the method's FLOP count (units x FLOPs per
    unit, see the table below).  Bytes: the method's own inputs the kernel must
    read from HBM and its outputs it must write (Q, K, V, O at the input
    width).  Intermediates (aggregated queries, Kt, Y, entropies) are NOT
    counted: a design that keeps them on chip or in L2 never pays for them, so
    HBM traffic above these bytes is overhead the roofline should expose.

      kernel          unit (count per launch)   FLOPs per unit          bytes per unit
      init_qt         (g, p, i)  G c1 b2        |p| d                   |p| d e   (Q rows)
      r_update        (g, k)     G b1           6 c1 b2^2 d (last step) 2 b2 d e  (K, V rows)
      l_update        (g, i, p)  G b2 c1        4 |p| b1 c2 d           |p| d e   (Q rows)
      l_output        (g, i, p)  G b2 c1        4 |p| b1 c2 d           2 |p| d e (Q in, O out)
      small_head      head g     G              the whole forward       4 N d e
    """
    G, N, d, b1, b2, c1, c2 = wl.heads, wl.N, wl.d, wl.b1, wl.b2, wl.c1, wl.c2
    e = elt_bytes(wl)
    io = G * N * d * e                          # one of Q, K, V or O
    if name.endswith("init_qt"):
        return G * N * d, io
    if name.endswith("r_update"):
        # logits + R K + R V: the timed launch is the last step's (it writes Y)
        return G * b1 * c1 * b2 * b2 * d * 2 * 3, 2 * io
    if name.endswith("l_output"):
        return G * N * b1 * c2 * d * 4, 2 * io
    if name == "tc_l_update":  # logits + L^T Q of a non-final step
        return G * N * b1 * c2 * d * 4, io
    if name.endswith("l_stats"):
        return G * N * b1 * c2 * d * 2, io
    if name.endswith("l_aggregate"):
        return G * N * b1 * c2 * d * 4, io
    if name == "small_head":  # the whole forward pass of small heads in one kernel
        return alg_flops(wl), alg_bytes(wl)
    if name == "permute_rows":  # aligned video layouts: q, k, v in, or the output back
        return 0, 2 * io * 2  # averaged over the two launches of a call (3 + 1 tensors)
    return 0, 0


def kernel_bound(name: str):
    # SIMT fp32 kernels, and the CUDA-core kernels of groups too small for the
    # tensor-core tiles (cc_*), against the FP32 lane rate
    return "alu" if name.startswith(("simt", "cc_")) else None


def roofline_for(name, tot_ms, launches, wl, peaks, peak_src, traffic):
    """Roofline entry of one kernel from its CUDA-event time.

    The bound is whichever of the kernel's algorithmic bytes (at the measured
    HBM copy bandwidth) and FLOPs (at the measured bf16 tensor rate, or the
    FP32 SIMT rate for SIMT kernels) takes longer.  Tensor-bound kernels are
    compared with the sustained bf16 rate, since the benchmark keeps them
    running back to back for over a second under the power cap.
    """
    avg_s = tot_ms / launches / 1e3
    fl, by = kernel_work(name, wl)
    t_mem = by / (peaks["hbm_gbs"] * 1e9)
    if kernel_bound(name) == "alu":
        peak_c, bound_c = ALU_FP32_TFLOPS, "alu"
        src_c = "derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz"
    else:
        peak_c = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        bound_c = "tensor"
        src_c = f"{peak_src} bf16 dense, sustained"
    t_cmp = fl / (peak_c * 1e12)
    if t_mem >= t_cmp:
        r = {"bound": "hbm", "achieved": by / avg_s / 1e9, "peak": peaks["hbm_gbs"],
             "unit": "GB/s"}
        r["peak_source"] = f"{peak_src} HBM copy"
    else:
        r = {"bound": bound_c, "achieved": fl / avg_s / 1e12, "peak": peak_c, "unit": "TFLOP/s"}
        r["peak_source"] = src_c
    r["frac"] = r["achieved"] / r["peak"]
    r["traffic"] = traffic
    r["algorithmic_bytes"] = by
    r["algorithmic_flops"] = fl
    r["traffic_over_algorithmic"] = (traffic / by) if (traffic and by) else None
    r["kernel"] = name
    r["kernel_ms"] = tot_ms / launches
    return r


# ---------------------------------------------------------------------------
# distributed helpers (also exercised by the gloo tests)
# ---------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def reduce_max(x: float, device) -> float:
    """Max of a scalar over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def job_value(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: work of all ranks divided by the slowest rank's time."""
    return units_per_rank * world / seconds


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


SMI_FIELDS = ["pci.bus_id", "clocks.sm", "clocks.max.sm", "power.draw",
              "clocks_event_reasons.active", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
REASON_COLS = {"clocks_event_reasons.hw_slowdown": "hw_slowdown",
               "clocks_event_reasons.hw_thermal_slowdown": "hw_thermal_slowdown",
               "clocks_event_reasons.sw_thermal_slowdown": "sw_thermal_slowdown",
               "clocks_event_reasons.sw_power_cap": "sw_power_cap"}


class ClockSampler:
    """Samples SM clock and throttle reasons with `nvidia-smi -lms` while the
    timed calls run, keeping the rows of this process's GPU (matched by PCI
    bus id, since nvidia-smi numbers GPUs differently from CUDA)."""

    def __init__(self, device_index: int, period_ms: int = 100, enabled: bool = True):
        self.period_ms = period_ms
        self.enabled = enabled
        self.err = "clock sampling disabled" if not enabled else None
        self.rows = []
        try:
            pr = torch.cuda.get_device_properties(device_index)
            self.bus = f"{int(pr.pci_bus_id):02X}:{int(pr.pci_device_id):02X}.0"  # "1B:00.0"
        except Exception as exc:
            self.enabled, self.err = False, repr(exc)

    def __enter__(self):
        import subprocess
        import tempfile
        if not self.enabled:
            return self
        self.tmp = tempfile.TemporaryFile(mode="w+")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(SMI_FIELDS), "--format=csv,noheader",
                 "-lms", str(self.period_ms)], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception as exc:
            self.enabled, self.err = False, repr(exc)
        return self

    def __exit__(self, *a):
        if not self.enabled:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except Exception:
            self.proc.kill()
        self.tmp.seek(0)
        for line in self.tmp:
            f = [x.strip() for x in line.split(",")]
            if len(f) == len(SMI_FIELDS) and f[0].upper().endswith(self.bus):
                self.rows.append(dict(zip(SMI_FIELDS, f)))
        self.tmp.close()

    def summary(self):
        if not self.enabled:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        def num(x):
            try:
                return float(x.split()[0])
            except Exception:
                return None
        mhz = [num(r["clocks.sm"]) for r in self.rows if num(r["clocks.sm"])]
        reasons = sorted({name for r in self.rows for col, name in REASON_COLS.items()
                          if r[col].lower() == "active"})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": num(self.rows[0]["clocks.max.sm"]) if self.rows else None,
                "reasons": reasons, "samples": len(self.rows),
                "power_w_max": max((num(r["power.draw"]) or 0) for r in self.rows)
                if self.rows else None,
                "window": "the timed calls plus the same calls repeated to >= 1 s"}


def traffic_for(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or
    None when the kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        f = line.split()
        if len(f) < 4 or f[0].startswith("#") or f[0] != kernel or f[1] != workload:
            continue
        kv = dict(x.split("=", 1) for x in f[2:] if "=" in x)
        src = os.path.join(ROOT, "structured_sub_quadratic_b200", "csrc", kv.get("src", ""))
        if not os.path.exists(src):
            return None
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if sha != kv.get("sha"):
            return None
        return float(kv["bytes"])
    return None


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(wl: Workload, budget_s: float, heads_per_run: int):
    """Time the float64 oracle on `heads_per_run` heads of wl, repeatedly,
    for about budget_s seconds; returns (TFLOP/s, seconds, heads done)."""
    from oracle import monarch_attention
    q, k, v = make_inputs(wl)
    hs = slice(0, heads_per_run)
    qn, kn, vn = (x.reshape(wl.heads, wl.N, wl.d)[hs].double().numpy() for x in (q, k, v))
    per_head = alg_flops(wl) / wl.heads
    done, t0 = 0, time.perf_counter()
    while True:
        monarch_attention(qn, kn, vn, wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
        done += heads_per_run
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return per_head * done / el / 1e12, el, done


def heads_for_budget(wl: Workload, target_s: float) -> int:
    """Heads of wl the oracle processes in about target_s (first estimate from one head)."""
    from oracle import monarch_attention
    q, k, v = make_inputs(Workload(**{**wl.__dict__, "B": 1, "H": 1}))
    t0 = time.perf_counter()
    monarch_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                      wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
    one = time.perf_counter() - t0
    return max(1, min(wl.heads, int(target_s / max(one, 1e-3))))


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------
def run_reference(args, wl):
    """The oracle as the reference arm, on the host cores (rank 0 only)."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    per_step_heads = heads_for_budget(wl, 0.5)
    per_head = alg_flops(wl) / wl.heads
    from oracle import monarch_attention
    q, k, v = make_inputs(wl)
    qn, kn, vn = (x.reshape(wl.heads, wl.N, wl.d)[:per_step_heads].double().numpy()
                  for x in (q, k, v))
    for _ in range(args.warmup):
        monarch_attention(qn, kn, vn, wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        monarch_attention(qn, kn, vn, wl.b1, wl.b2, wl.T, wl.c1, wl.c2)
    el = time.perf_counter() - t0
    value = per_head * per_step_heads * args.steps / el / 1e12
    sample = (f"{per_step_heads} of {wl.heads} heads of the workload per step "
              f"(float64 numpy oracle)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, None),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl: Workload, l2_note, layout=None):
    cfg = {"workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "b1": wl.b1, "b2": wl.b2,
           "d": wl.d, "T": wl.T, "c1": wl.c1, "c2": wl.c2, "inputs": wl.kind, "seed": wl.seed}
    if wl.latent:
        cfg["latent_fhw"] = list(wl.latent)
    if layout:
        cfg["layout"] = f"({layout})"

    if l2_note:
        cfg["l2"] = l2_note
    return cfg


def run_native(args, wl):
    from structured_sub_quadratic_b200 import api
    rank, local_rank, world = dist_env()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device,
                                timeout=datetime.timedelta(seconds=300))
    api.load_library()
    stream = torch.cuda.current_stream(device)
    log("library loaded")

    # rotating device-resident input sets, together several times the L2
    io_in = 3 * wl.heads * wl.N * wl.d * elt_bytes(wl)
    n_sets = max(1, min(16, math.ceil(4 * L2_BYTES / io_in)))
    sets = []
    for s in range(n_sets):
        w = Workload(**{**wl.__dict__, "seed": wl.seed + 1000 * rank + s})
        q, k, v = (x.to(device) for x in make_inputs(w))
        sets.append((q, k, v, torch.empty_like(q)))
    if n_sets == 1:
        l2_note = (f"one device-resident input set whose Q/K/V ({io_in / 2**20:.0f} MiB) "
                   f"exceed the 126 MiB L2")
    else:
        l2_note = (f"inputs rotate over {n_sets} device-resident sets "
                   f"({n_sets * io_in / 2**20:.0f} MiB of Q/K/V > 126 MiB L2)")

    def step(s):
        q, k, v, o = sets[s % n_sets]
        if args.layout:
            api.monarch_attn_fwd_video(q, k, v, *wl.latent, args.layout, wl.T, wl.c1, wl.c2,
                                       out=o, stream=stream)
        else:
            api.monarch_attn_fwd(q, k, v, wl.b1, wl.b2, wl.T, wl.c1, wl.c2, out=o, stream=stream)

    log(f"{n_sets} input sets on device")
    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize(device)
    api.check(stream)
    log("warm-up done")
    launches_per_call = api.last_launches()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank, enabled=not args.no_clocks) as clk:
        barrier(device)
        torch.cuda.synchronize(device)
        ev0.record(stream)
        for s in range(args.steps):
            step(s)
        ev1.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        ms_local = ev0.elapsed_time(ev1)
        # keep the same calls running for >= 1 s so the sampler sees the load
        t_end = time.perf_counter() + max(0.0, 1.0 - ms_local / 1e3)
        s = 0
        while time.perf_counter() < t_end:
            for _ in range(20):
                step(s)
                s += 1
            torch.cuda.synchronize(device)
    api.check(stream)
    log(f"timed region done: {ms_local:.3f} ms; clocks {clk.summary()}")
    ms = reduce_max(ms_local, device)
    flops = alg_flops(wl)
    value = job_value(flops * args.steps, world, ms / 1e3) / 1e12

    # per-kernel device time (CUDA events around every launch, same stream)
    api.timing_read()
    api.timing_enable(True)
    for s in range(args.steps):
        step(s)
    torch.cuda.synchronize(device)
    per_kernel = api.timing_read()
    api.timing_enable(False)
    log(f"per-kernel timing: {per_kernel}")
    roofline = None
    peaks, peak_src = load_peaks()
    if per_kernel:
        name, (tot_ms, n) = max(per_kernel.items(), key=lambda kv: kv[1][0])
        roofline = roofline_for(name, tot_ms, n, wl, peaks, peak_src,
                                traffic_for(name, args.workload))
        total = sum(x[0] for x in per_kernel.values())
        roofline["kernels"] = {
            k: {"ms": t / c, "launches_per_call": c / args.steps, "share": t / total,
                "frac": roofline_for(k, t, c, wl, peaks, peak_src, None)["frac"],
                "bound": roofline_for(k, t, c, wl, peaks, peak_src, None)["bound"]}
            for k, (t, c) in per_kernel.items()}

    # end to end through the public API with host buffers, copies inside the timed region:
    # the host-buffer C-ABI call, or (aligned video layouts) pinned-host copies around the
    # video-layout call
    q, k, v, o = sets[0]
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    e2e_steps = max(1, min(args.steps, 50))

    def e2e_call():
        if args.layout:
            for dst, src in ((q, qh), (k, kh), (v, vh)):
                dst.copy_(src, non_blocking=True)
            api.monarch_attn_fwd_video(q, k, v, *wl.latent, args.layout, wl.T, wl.c1, wl.c2,
                                       out=o, stream=stream)
            oh.copy_(o, non_blocking=True)
            torch.cuda.current_stream(device).synchronize()
        else:
            api.monarch_attn_fwd_host(qh, kh, vh, oh, wl.b1, wl.b2, wl.T, wl.c1, wl.c2,
                                      stream=stream)

    e2e_call()
    barrier(device)
    torch.cuda.synchronize(device)
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_call()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    e2e_ms = reduce_max(ev0.elapsed_time(ev1) / e2e_steps, device)
    e2e_value = job_value(flops, world, e2e_ms / 1e3) / 1e12
    log(f"e2e done: {e2e_ms:.3f} ms/step")
    io_elt = wl.heads * wl.N * wl.d * elt_bytes(wl)

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nh = heads_for_budget(wl, 2.0)
        log(f"cpu baseline: {nh} heads per oracle call")
        val, el, done = oracle_sample(wl, args.cpu_seconds, nh)
        cpu_baseline = {"value": val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                        "sample": f"{done} heads of the workload ({nh} per oracle call, "
                                  f"{el:.1f} s, float64 numpy)"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f32",
        "data": "synthetic", "config": workload_config(wl, l2_note, args.layout),
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": 3 * io_elt, "d2h_bytes_per_step": io_elt},
        "gpu_launches": launches_per_call * args.steps,
        "roofline": roofline,
        "cpu_baseline": cpu_baseline,
        # whole-call figures for context (not a roofline of one kernel)
        "context": {
            "path_hbm_frac": (alg_bytes(wl) / (ms / args.steps / 1e3) / 1e9) / peaks["hbm_gbs"],
            "path_tensor_frac_sustained":
                (flops / (ms / args.steps / 1e3) / 1e12)
                / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
            # the 4 N^2 d FLOPs dense softmax attention would need on this shape, over the
            # measured time: a ratio of the method's savings, NOT a throughput of this chip
            "dense_attention_equivalent_tflops":
                wl.heads * 4.0 * wl.N * wl.N * wl.d / (ms / args.steps / 1e3) / 1e12,
        },
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(device)
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="720p", choices=sorted(WORKLOADS),
                    help="default: the 720p video config, the largest single-GPU workload")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true", help="skip the clock sampler")
    ap.add_argument("--layout", default=None,
                    choices=["fh,w", "w,fh", "f,hw", "hw,f", "fw,h", "h,fw"],
                    help="video workloads: aligned block layout of the latent (raster-order "
                         "inputs through the video-layout entry point)")
    ap.add_argument("--heads", type=int, default=None,
                    help="override H (profiling a smaller case of the same shape)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.heads is not None:
        wl = Workload(**{**wl.__dict__, "H": args.heads, "name": f"{wl.name} [H={args.heads}]"})
    if args.layout:
        if not wl.latent:
            ap.error("--layout needs a video workload (480p or 720p)")
        size = dict(zip("fhw", wl.latent))
        rows, cols = args.layout.split(",")
        b1 = math.prod(size[a] for a in rows)
        wl = Workload(**{**wl.__dict__, "b1": b1, "b2": wl.N // b1,
                         "name": f"{wl.name} blocks ({args.layout})=({b1},{wl.N // b1})"})
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_native(args, wl)


if __name__ == "__main__":
    sys.exit(main())
