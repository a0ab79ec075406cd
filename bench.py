#!/usr/bin/env python
"""Benchmark of the gated sliding-window attention core on B200.

One step = one pass of the hot path over one batch of synthetic input held in
HBM.  The headline line times swa_fwd on the ZGCM-1 layer-shape prefill
workload (B=4, T=4096, 32 query / 8 KV heads, head_dim 128, window 128,
rot_dim 42): norm, RoPE, windowed GQA attention and the gate all run inside
the one fused kernel launch that forms the step.  Secondary workloads (the
long-context forward, training forward+backward and the 27-layer decode step)
are timed the same way and reported under "secondary".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl swa|reference]

For N > 1 launch with torchrun: each rank runs its own batch (the batch rows
are independent problems, so there is no data-path collective; scaling is
weak) and the reported time is the maximum over ranks.  `--impl reference`
times the fp64 CPU oracle on bounded samples of the same workload (rank 0
only).
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402


def FWD_BYTES_PER_TOKEN(c):
    """Algorithmic HBM bytes per token of the forward: read q, g, k, v; write o."""
    return (3 * c.Hq + 2 * c.Hkv) * c.D * 2


def BWD_BYTES_PER_TOKEN(c):
    """Backward: read q, g, dO, k, v and lse; write dq, dg, dk, dv."""
    return (3 * c.Hq + 2 * c.Hkv) * c.D * 2 + c.Hq * 4 + (2 * c.Hq + 2 * c.Hkv) * c.D * 2


def band_keys(T, W):
    """sum_i min(i+1, W) for one sequence of T tokens."""
    full = max(T - W + 1, 0)
    ramp = min(T, W - 1)
    return full * W + ramp * (ramp + 1) // 2


def fwd_flops(c):
    return 4 * c.D * c.Hq * band_keys(c.T, c.W) * c.B


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured (MEASURED_PEAKS.json)"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback (profiling recipe)"}


def kernel_source_digest(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "hybrid_sliding_window_gated_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(profile_name, files):
    """dram bytes per launch from a committed ncu summary, or None if the kernel
    sources changed since it was captured."""
    path = os.path.join(ROOT, "profiles", profile_name)
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if "=" in line and not line.lstrip().startswith("#"):
                k, v = (s.strip() for s in line.split("=", 1))
                vals[k] = v
    if vals.get("kernel_sources_sha256_16") != kernel_source_digest(files):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a thread."""

    def __init__(self, device_index, period_s=0.005):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = torch.cuda.get_device_properties(device_index).uuid
            self.h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == str(uuid).replace("GPU-", ""):
                    self.h = h
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report no clocks rather than fail
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        nv = self.nv
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "applications_clocks_setting": getattr(nv, "nvmlClocksEventReasonApplicationsClocksSetting", 0x2),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sync_boost": getattr(nv, "nvmlClocksEventReasonSyncBoost", 0x10),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if not inside:  # timed region shorter than one sampling period
            inside = self.samples[-5:]
            window = "last samples after the timed region"
        mhz = [s[1] for s in inside]
        active = set()
        for s in inside:
            for n, bit in names.items():
                if s[2] & bit and n != "gpu_idle":
                    active.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(active), "samples": len(inside), "window": window}


# ----------------------------------------------------------------- timing

def max_over_ranks(ms, world):
    """The slowest rank's device time: every rank takes part (same collective
    in every rank's sequence); the tensor lives where the backend wants it."""
    if world <= 1:
        return ms
    on_gpu = torch.distributed.get_backend() == "nccl"
    t = torch.tensor([ms], dtype=torch.float64, device="cuda" if on_gpu else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, world, steps, ms):
    """Whole-job units per second: every rank processed `units_per_rank` per
    step (weak scaling), timed by the slowest rank."""
    return units_per_rank * world * steps / (ms / 1e3)


def timed_loop(step_fns, steps, warmup, stream, world, sampler=None, per_launch=None):
    """Run warmup steps, then time `steps` steps between barriers on `stream`.

    step_fns: list of callables, one per rotating input set.  Returns
    (total_ms max over ranks, per-launch mean ms of the measured kernel, t0, t1).
    """
    for i in range(warmup):
        step_fns[i % len(step_fns)]()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launch_evs = []
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for i in range(steps):
            if per_launch is not None:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                step_fns[i % len(step_fns)]()
                b.record(stream)
                launch_evs.append((a, b))
            else:
                step_fns[i % len(step_fns)]()
        ev1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    per = None
    if launch_evs:
        per = sum(a.elapsed_time(b) for a, b in launch_evs) / len(launch_evs)
    return ms, per, t0, t1


# ------------------------------------------------------------- workloads

def fwd_workload(swa, cfg, device, n_sets=2, lse=False):
    sets = []
    for s in range(n_sets):
        inp = workloads.prefill_inputs(cfg, device=device, seed=cfg.seed + 100 * s,
                                       with_grad_out=False)
        inp["o"] = torch.empty_like(inp["q"])
        inp["lse"] = torch.empty((cfg.B, cfg.Hq, cfg.T), dtype=torch.float32, device=device) \
            if lse else None
        sets.append(inp)

    def mk(inp):
        def step():
            swa.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["wq"], inp["wk"], window=cfg.W,
                    rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps, out=inp["o"], lse=inp["lse"])
        return step
    return [mk(x) for x in sets], sets


def e2e_fwd(swa, cfg, device, steps, warmup, stream, world):
    """Same metric through the public call with pinned host buffers: H2D of the
    step's inputs, swa_fwd, D2H of the output, all inside the timed region."""
    host = workloads.prefill_inputs(cfg, device="cpu", with_grad_out=False)
    host = {k: v.pin_memory() for k, v in host.items()}
    out_host = torch.empty(host["q"].shape, dtype=torch.bfloat16).pin_memory()
    dev = {k: torch.empty_like(v, device=device) for k, v in host.items()}
    o = torch.empty_like(dev["q"])
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def step():
        for k in host:
            dev[k].copy_(host[k], non_blocking=True)
        swa.fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["wq"], dev["wk"], window=cfg.W,
                rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps, out=o)
        out_host.copy_(o, non_blocking=True)
    ms, _, _, _ = timed_loop([step], steps, warmup, stream, world)
    return ms, h2d, d2h


def oracle_pass(oracle, inp, cfg):
    """One pass of the fp64 oracle over the whole forward workload (every batch
    row, token and head), row by row so lse is not materialised."""
    for b in range(cfg.B):
        oracle.fwd_rows(inp["q"], inp["k"], inp["v"], inp["g"], inp["wq"], inp["wk"], b, 0, cfg.T,
                        W=cfg.W, R=cfg.R, base=cfg.base, eps=cfg.eps)


def cpu_baseline_fwd(cfg, target_s=10.0):
    """Time the fp64 oracle, as it stands, on this host's cores: whole passes
    over the workload, repeated until at least target_s seconds have run."""
    import oracle
    inp = workloads.prefill_inputs(cfg, device="cpu", with_grad_out=False)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_pass(oracle, inp, cfg)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            break
    tokens = reps * cfg.B * cfg.T
    return {"value": tokens / dt, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"the whole {cfg.name} workload ({cfg.B * cfg.T} query tokens x {cfg.Hq} "
                      f"heads), {reps} passes, fp64, {dt:.1f} s"}


# ---------------------------------------------------------------- main

def run_swa(args, rank, world, device):
    import hybrid_sliding_window_gated_b200 as swa
    from hybrid_sliding_window_gated_b200 import build as swa_build
    if rank == 0:
        swa_build.build()
    if world > 1:
        torch.distributed.barrier()
    swa.lib()
    peaks = load_peaks()
    cfg = workloads.LAYER
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(torch.cuda.current_device())

    steps_fns, _ = fwd_workload(swa, cfg, device)
    # Launches timed one by one (an event pair around each): the events keep
    # each launch from overlapping its prologue with the previous one's tail,
    # so this is the kernel's isolated duration, reported beside the figure.
    _, isolated_ms, _, _ = timed_loop(steps_fns, max(args.steps, 10), args.warmup, stream,
                                      world, per_launch=True)
    # The timed region (K steps) is repeated until about half a second has
    # run, so the clock samples come from inside the regions; the reported
    # time is the median region.  The repeat count is agreed across ranks,
    # since each region ends in a collective.
    sampler.start()
    ms, _, t0, _ = timed_loop(steps_fns, args.steps, args.warmup, stream, world)
    regions = [ms]
    n_regions = int(max_over_ranks(float(max(1, math.ceil(500.0 / max(ms, 1e-3)))), world))
    for _ in range(n_regions - 1):
        r, _, _, _ = timed_loop(steps_fns, args.steps, 0, stream, world)
        regions.append(r)
    t1 = time.perf_counter()
    sampler.stop()
    clocks = sampler.summary(t0, t1)
    ms = statistics.median(regions)

    tokens_per_rank = cfg.B * cfg.T
    value = aggregate_throughput(tokens_per_rank, world, args.steps, ms)
    bytes_launch = FWD_BYTES_PER_TOKEN(cfg) * tokens_per_rank
    # The timed region launches only swa_fwd_kernel, one per step: its average
    # launch duration is the region's event time over the launches.
    per_launch_ms = ms / args.steps
    achieved = bytes_launch / (per_launch_ms / 1e3) / 1e9
    traffic = committed_traffic("swa_fwd_kernel_layer_shape.txt", ["fwd.cu", "ptx.cuh", "swa_internal.h"])

    e2e_ms, h2d, d2h = e2e_fwd(swa, cfg, device, max(3, min(args.steps, 10)), 2, stream, world)
    e2e_value = tokens_per_rank * world / (e2e_ms / max(3, min(args.steps, 10)) / 1e3)

    line = {
        "metric": "gated-SWA forward tokens/s (layer-shape prefill)",
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded randn, ZGCM-1 layer shapes)",
        "config": {"workload": cfg.name, "B": cfg.B, "T": cfg.T, "Hq": cfg.Hq, "Hkv": cfg.Hkv,
                   "head_dim": cfg.D, "window": cfg.W, "rot_dim": cfg.R, "rope_base": cfg.base,
                   "parallelism": f"independent batches x{world}",
                   "l2": "two rotating input sets of 470 MB each (> 126 MB L2)"},
        "gpu_launches": args.steps,
        "timed_regions": {"count": len(regions), "ms_min": round(min(regions), 4),
                          "ms_median": round(ms, 4), "ms_max": round(max(regions), 4),
                          "sm_mhz_median": clocks.get("sm_mhz")},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": traffic, "kernel": "swa_fwd_kernel",
                     "algorithmic_bytes_per_launch": bytes_launch,
                     "launch_ms": round(per_launch_ms, 5),
                     "launch_ms_isolated": round(isolated_ms, 5),
                     "frac_isolated": round(bytes_launch / (isolated_ms / 1e3) / 1e9
                                            / peaks["hbm_gbs"], 4),
                     "peak_source": peaks["source"] + ", hbm_gbs (burst copy)"},
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clocks,
    }
    if not args.no_secondary:
        line["secondary"] = secondary(swa, args, world, device, stream, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_fwd(cfg)
    return line


def secondary(swa, args, world, device, stream, peaks):
    out = {}
    cfg = workloads.LONG
    fns, sets = fwd_workload(swa, cfg, device, n_sets=1)
    steps = max(3, min(args.steps, 10))
    ms, per, _, _ = timed_loop(fns, steps, 2, stream, world, per_launch=True)
    b = FWD_BYTES_PER_TOKEN(cfg) * cfg.B * cfg.T
    out["long_context_fwd"] = {
        "workload": cfg.name, "tokens_per_s": round(cfg.B * cfg.T * world / (ms / steps / 1e3), 1),
        "ms_per_step": round(ms / steps, 4),
        "achieved_GBps": round(b / (per / 1e3) / 1e9, 1),
        "frac_of_measured_hbm": round(b / (per / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "l2": "7.5 GB per step (> L2)"}
    del fns, sets
    torch.cuda.empty_cache()
    out["train_fwd_bwd"] = train_bench(swa, args, world, device, stream, peaks)
    out["decode_step"] = decode_bench(swa, args, world, device, stream, peaks)
    out["prefill_to_ring"] = ring_bench(swa, args, world, device, stream, peaks)
    out["fp8_fwd"] = fp8_fwd_bench(swa, args, world, device, stream, peaks)
    out["global_prefill"] = global_prefill_bench(swa, args, world, device, stream, peaks)
    out["global_decode_step"] = global_decode_bench(swa, args, world, device, stream, peaks)
    return out


def FP8_FWD_BYTES_PER_TOKEN(c):
    """The forward with E4M3 q, k, v: one byte each for q, k, v; g and o bf16."""
    return (c.Hq + 2 * c.Hkv) * c.D + 2 * c.Hq * c.D * 2


def fp8_fwd_bench(swa, args, world, device, stream, peaks):
    """swa_fwd_fp8 on the layer shape (4 x 4096): q, k, v in E4M3 with one factor
    each; two rotating input sets (> L2)."""
    cfg = workloads.LAYER
    sets = []
    for s in range(2):
        x = workloads.fp8_prefill_inputs(cfg, device=device, seed=cfg.seed + 100 * s)
        x["o"] = torch.empty(x["g"].shape, dtype=torch.bfloat16, device=device)
        sets.append(x)

    def mk(x):
        return lambda: swa.fwd_fp8(x["q8"], x["k8"], x["v8"], x["qkv_scale"], x["g"], x["wq"],
                                   x["wk"], rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps,
                                   out=x["o"])
    steps = max(5, min(args.steps, 20))
    ms, _, _, _ = timed_loop([mk(x) for x in sets], steps, 3, stream, world)
    b = FP8_FWD_BYTES_PER_TOKEN(cfg) * cfg.B * cfg.T
    gbs = b / (ms / steps / 1e3) / 1e9
    res = {"workload": cfg.name + ", q/k/v in FP8 E4M3",
           "tokens_per_s": round(cfg.B * cfg.T * world / (ms / steps / 1e3), 1),
           "ms_per_step": round(ms / steps, 5),
           "algorithmic_bytes_per_step": b,
           "achieved_GBps": round(gbs, 1),
           "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    del sets
    torch.cuda.empty_cache()
    return res


def global_fwd_flops(c):
    """QK^T and PV over the causal triangle: 4 D Hq sum_i (i + 1) per sequence."""
    return 4 * c.D * c.Hq * c.T * (c.T + 1) // 2 * c.B


def global_prefill_bench(swa, args, world, device, stream, peaks):
    """A global layer's causal prefill (swa_global_fwd: cache writer + tcgen05
    attention) on 1 x 16384, 32 / 8 heads.  Tensor-bound: 2.2e12 band FLOPs
    against 0.3 GB of traffic."""
    cfg = workloads.GLOBAL_PREFILL
    d = workloads.prefill_inputs(cfg, device=device, with_grad_out=False)
    kc = torch.empty((cfg.B, cfg.Hkv, cfg.T, cfg.D), dtype=torch.bfloat16, device=device)
    vc = torch.empty_like(kc)
    o = torch.empty_like(d["q"])

    def step():
        swa.global_fwd(d["q"], d["k"], d["v"], d["wq"], d["wk"], kc, vc, rot_dim=cfg.R,
                       rope_base=cfg.base, eps=cfg.eps, out=o)
    steps = max(3, min(args.steps, 10))
    ms, _, _, _ = timed_loop([step], steps, 3, stream, world)
    fl = global_fwd_flops(cfg)
    tf = fl / (ms / steps / 1e3) / 1e12
    res = {"workload": cfg.name,
           "tokens_per_s": round(cfg.B * cfg.T * world / (ms / steps / 1e3), 1),
           "ms_per_step": round(ms / steps, 4),
           "algorithmic_flops_per_step": fl,
           "achieved_TFLOPs": round(tf, 1),
           "frac_of_measured_bf16": round(tf / peaks["bf16_tflops"], 4),
           "frac_of_measured_bf16_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
           "bound": "tensor", "launches_per_step": 2}
    del d, kc, vc, o
    torch.cuda.empty_cache()
    return res


def global_decode_bench(swa, args, world, device, stream, peaks):
    """A decode step of the 5 global layers: one swa_global_decode_step per
    layer over its own [64, 8, 32768, 128] K and V caches (8.6 GB each), at
    positions uniform in [1, 32768).  HBM-bound: the K and V of positions
    0 .. pos, plus q, k, v, o rows."""
    cfg = workloads.GLOBAL_DECODE
    layers = [workloads.global_decode_layer_inputs(cfg, l, device=device)
              for l in range(cfg.layers)]
    outs = [torch.empty_like(x["q"]) for x in layers]
    ws = torch.empty(swa.global_decode_workspace_size(cfg.N, cfg.Hq, cfg.Hkv, cfg.cap),
                     dtype=torch.uint8, device=device)

    def step():
        for x, o in zip(layers, outs):
            swa.global_decode_step(x["pos"], x["q"], x["k"], x["v"], x["wq"], x["wk"],
                                   x["k_cache"], x["v_cache"], rot_dim=cfg.R, rope_base=cfg.base,
                                   eps=cfg.eps, out=o, workspace=ws)
    steps = max(3, min(args.steps, 10))
    ms, _, _, _ = timed_loop([step], steps, 3, stream, world)
    kv_row = cfg.Hkv * cfg.D * 2
    b = 0
    for x in layers:  # keys 0..pos read from both caches; new k, v written; q read, o written
        b += int((x["pos"] + 1).sum().item()) * kv_row * 2 + cfg.N * (2 * kv_row + 2 * kv_row
                                                                     + 2 * cfg.Hq * cfg.D * 2)
    gbs = b / (ms / steps / 1e3) / 1e9
    res = {"workload": cfg.name,
           "tokens_per_s": round(cfg.N * world / (ms / steps / 1e3), 1),
           "ms_per_step": round(ms / steps, 4),
           "algorithmic_bytes_per_step": b,
           "achieved_GBps": round(gbs, 1),
           "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 4),
           "launches_per_step": 3 * cfg.layers,
           "note": "positions fixed across steps: each step rewrites the same cache slots"}
    del layers, outs, ws
    torch.cuda.empty_cache()
    return res


def train_bench(swa, args, world, device, stream, peaks):
    """Training step of the layer core on the training shape: swa_fwd (with
    lse) then swa_bwd; inputs 1x16384 are above L2 (2.1 GB live)."""
    cfg = workloads.TRAIN
    d = workloads.prefill_inputs(cfg, device=device, with_grad_out=True)
    o = torch.empty_like(d["q"])
    lse = torch.empty((cfg.B, cfg.Hq, cfg.T), dtype=torch.float32, device=device)
    grads = (torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"]),
             torch.empty_like(d["g"]), torch.zeros(cfg.D, device=device),
             torch.zeros(cfg.D, device=device))
    ws = torch.empty(swa.bwd_workspace_size(cfg.B, cfg.T, cfg.Hq, cfg.Hkv), dtype=torch.uint8,
                     device=device)

    def fwd():
        swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], rope_base=cfg.base,
                out=o, lse=lse)

    def bwd():
        swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"],
                rope_base=cfg.base, workspace=ws, grads=grads)

    def step():
        fwd()
        bwd()
    steps = max(3, min(args.steps, 10))
    ms, _, _, _ = timed_loop([step], steps, 3, stream, world)
    ms_b, _, _, _ = timed_loop([bwd], steps, 3, stream, world)
    tok = cfg.B * cfg.T
    b_fb = (FWD_BYTES_PER_TOKEN(cfg) + cfg.Hq * 4 + BWD_BYTES_PER_TOKEN(cfg)) * tok
    b_b = BWD_BYTES_PER_TOKEN(cfg) * tok
    res = {"workload": cfg.name,
           "tokens_per_s": round(tok * world / (ms / steps / 1e3), 1),
           "ms_per_step": round(ms / steps, 4),
           "algorithmic_bytes_per_step": b_fb,
           "achieved_GBps": round(b_fb / (ms / steps / 1e3) / 1e9, 1),
           "frac_of_measured_hbm": round(b_fb / (ms / steps / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
           "bwd_ms": round(ms_b / steps, 4),
           "bwd_frac_of_measured_hbm":
               round(b_b / (ms_b / steps / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
           "launches_per_step": 3}
    del d, o, lse, grads, ws
    torch.cuda.empty_cache()
    return res


def DECODE_BYTES_PER_SEQ_LAYER(c):
    """Algorithmic HBM bytes of one (sequence, layer) decode: the W-1 older ring
    slots of K and V, the new k and v, their slot writes, and q, g, o."""
    kv_row = c.Hkv * c.D * 2
    return (c.W - 1) * kv_row * 2 + 2 * kv_row + 2 * kv_row + 3 * c.Hq * c.D * 2


def decode_bench(swa, args, world, device, stream, peaks):
    """A decode step of the whole model's window layers: one swa_decode_step per
    layer, each over its own [N, Hkv, 128, 128] K and V rings (3.5 GB > L2)."""
    cfg = workloads.DECODE
    layers = [workloads.decode_layer_inputs(cfg, l, device=device) for l in range(cfg.layers)]
    outs = [torch.empty_like(x["q"]) for x in layers]

    def step():
        for x, o in zip(layers, outs):
            swa.decode_step(x["pos"], x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"],
                            x["k_cache"], x["v_cache"], rot_dim=cfg.R, rope_base=cfg.base,
                            eps=cfg.eps, out=o)
    steps = max(5, min(args.steps, 20))
    ms, per, _, _ = timed_loop([step], steps, 3, stream, world, per_launch=True)
    b = DECODE_BYTES_PER_SEQ_LAYER(cfg) * cfg.N * cfg.layers
    res = {"workload": cfg.name,
           "tokens_per_s": round(cfg.N * world / (ms / steps / 1e3), 1),
           "ms_per_step": round(ms / steps, 4),
           "algorithmic_bytes_per_step": b,
           "achieved_GBps": round(b / (per / 1e3) / 1e9, 1),
           "frac_of_measured_hbm": round(b / (per / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
           "launches_per_step": cfg.layers,
           "note": "positions fixed across steps: each step rewrites the same ring slots"}
    del layers, outs
    torch.cuda.empty_cache()
    return res


def ring_bench(swa, args, world, device, stream, peaks):
    """The prefill -> ring handoff for the decode batch: 256 sequences with a
    256-token prefix, 8 KV heads; the last 128 positions' k and v are read and
    the K and V rings written (128 B x 4 per element row: 268 MB per call over
    two rotating input sets of 536 MB each, > L2)."""
    N, T, Hkv, Hq, D, W = 256, 256, 8, 32, 128, 128
    gen = torch.Generator(device="cpu").manual_seed(7)
    sets = []
    for _ in range(2):
        k = torch.randn((N, T, Hkv, D), generator=gen).to(torch.bfloat16).to(device)
        v = torch.randn((N, T, Hkv, D), generator=gen).to(torch.bfloat16).to(device)
        kc = torch.empty((N, Hkv, W, D), dtype=torch.bfloat16, device=device)
        sets.append((k, v, kc, torch.empty_like(kc)))
    wk = (1.0 + 0.1 * torch.randn(D, generator=gen)).to(device)

    def mk(x):
        return lambda: swa.prefill_to_ring(x[0], x[1], wk, x[2], x[3], Hq=Hq, rope_base=1e7)
    steps = max(5, min(args.steps, 20))
    ms, per, _, _ = timed_loop([mk(x) for x in sets], steps, 3, stream, world, per_launch=True)
    b = 4 * N * Hkv * W * D * 2  # read k, v rows; write the K and V ring slots
    res = {"workload": f"prefill -> ring handoff, {N} sequences x {T} tokens, {Hkv} kv heads",
           "ms_per_call": round(ms / steps, 5),
           "algorithmic_bytes_per_call": b,
           "achieved_GBps": round(b / (per / 1e3) / 1e9, 1),
           "frac_of_measured_hbm": round(b / (per / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}
    del sets
    torch.cuda.empty_cache()
    return res


def run_profile(args, device):
    """Warmup + steps calls of one entry point, nothing else, so that a
    profiler sees a short, predictable launch list: `fwd` on the layer-shape
    workload, `decode` on one layer of the decode workload, `bwd` (with the
    forward that produces its lse) on the training shape, `ring` on the
    prefill -> ring handoff of the decode batch, `gfwd` on the global-layer
    prefill, `gdec` on 16 sequences of one global layer's decode."""
    import hybrid_sliding_window_gated_b200 as swa
    which = args.profile
    if which == "fwd":
        cfg = workloads.LAYER
        fns, _ = fwd_workload(swa, cfg, device)
    elif which == "decode":
        cfg = workloads.DECODE
        x = workloads.decode_layer_inputs(cfg, 0, device=device)
        o = torch.empty_like(x["q"])
        fns = [lambda: swa.decode_step(x["pos"], x["q"], x["k"], x["v"], x["g"], x["wq"], x["wk"],
                                       x["k_cache"], x["v_cache"], rot_dim=cfg.R,
                                       rope_base=cfg.base, eps=cfg.eps, out=o)]
    elif which == "gfwd":
        cfg = workloads.GLOBAL_PREFILL
        d = workloads.prefill_inputs(cfg, device=device, with_grad_out=False)
        kc = torch.empty((cfg.B, cfg.Hkv, cfg.T, cfg.D), dtype=torch.bfloat16, device=device)
        vc = torch.empty_like(kc)
        fns = [lambda: swa.global_fwd(d["q"], d["k"], d["v"], d["wq"], d["wk"], kc, vc,
                                      rot_dim=cfg.R, rope_base=cfg.base, eps=cfg.eps)]
    elif which == "gdec":
        # 16 of the 64 sequences (2.1 GB of caches), so a full capture stays small
        cfg = workloads.GLOBAL_DECODE
        x = workloads.global_decode_layer_inputs(cfg, 0, device=device)
        x = {k: (v[:16].contiguous() if v.dim() > 1 or k == "pos" else v) for k, v in x.items()}
        o = torch.empty_like(x["q"])
        fns = [lambda: swa.global_decode_step(x["pos"], x["q"], x["k"], x["v"], x["wq"], x["wk"],
                                              x["k_cache"], x["v_cache"], rot_dim=cfg.R,
                                              rope_base=cfg.base, eps=cfg.eps, out=o)]
    elif which == "ring":
        cfg = workloads.custom_prefill(256, 256, 32, 8, base=1e7, seed=7)
        gen = torch.Generator(device="cpu").manual_seed(7)
        k = torch.randn((256, 256, 8, 128), generator=gen).to(torch.bfloat16).to(device)
        v = torch.randn((256, 256, 8, 128), generator=gen).to(torch.bfloat16).to(device)
        wk = (1.0 + 0.1 * torch.randn(128, generator=gen)).to(device)
        kc = torch.empty((256, 8, 128, 128), dtype=torch.bfloat16, device=device)
        vc = torch.empty_like(kc)
        fns = [lambda: swa.prefill_to_ring(k, v, wk, kc, vc, Hq=32, rope_base=1e7)]
    else:
        cfg = workloads.TRAIN
        d = workloads.prefill_inputs(cfg, device=device, with_grad_out=True)
        o, lse = swa.fwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], rope_base=cfg.base,
                         want_lse=True)
        fns = [lambda: swa.bwd(d["q"], d["k"], d["v"], d["g"], d["wq"], d["wk"], lse, d["dO"],
                               rope_base=cfg.base)]
    for i in range(args.warmup + args.steps):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    code, site = swa.get_last_device_error()
    return {"profile": cfg.name, "entry": which, "launches": args.warmup + args.steps,
            "device_error": code}


def run_reference(args, rank, world):
    """The fp64 oracle on bounded samples, as the reference arm (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    cfg = workloads.LAYER
    inp = workloads.prefill_inputs(cfg, device="cpu", with_grad_out=False)

    def step(i):
        oracle_pass(oracle, inp, cfg)  # one step = the whole workload, as on the GPU
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    value = cfg.B * cfg.T * args.steps / dt
    return {
        "metric": "gated-SWA forward tokens/s (layer-shape prefill)", "impl": "reference",
        "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded randn, ZGCM-1 layer shapes)",
        "config": {"workload": cfg.name, "B": cfg.B, "T": cfg.T, "Hq": cfg.Hq, "Hkv": cfg.Hkv,
                   "head_dim": cfg.D, "window": cfg.W, "rot_dim": cfg.R, "rope_base": cfg.base,
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": oracle.threads(),
                         "kind": "oracle",
                         "sample": f"each step the whole {cfg.name} workload "
                                   f"({cfg.B * cfg.T} query tokens x {cfg.Hq} heads), fp64"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["swa", "reference"], default="swa")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["fwd", "decode", "bwd", "ring", "gfwd", "gdec"],
                    default=None,
                    help="only warmup + steps calls of one entry point (for ncu)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120),
                                             device_id=device)
    if args.profile is not None:
        line = run_profile(args, device)
    else:
        line = run_swa(args, rank, world, device)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
