#!/usr/bin/env python
"""Benchmark of the fused MoE top-k gating operator on B200.

One step = one fused gating call (logits -> top-k -> softmax, one kernel launch)
over one batch of synthetic tokens.  Default workload: the training-microbatch
router, T=65536 tokens, H=7168, E=256 experts, k=8 (hidden 940 MB > L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

``--precision fp8`` times the FP8 (E4M3) entry point on the workload's inputs
quantized per token (hidden) and per expert (gate).  ``--op route`` times the routing metadata (per-expert offsets, the expert-grouped
order and each assignment's position) of seeded ids of the workload's T x k
shape; ``--op gating_route`` times gating and the routing of its ids in one call (the counts per expert
taken by the gating kernel), beside the gating alone and the two separate calls.

Prints ONE JSON line on rank 0.  With N > 1 (torchrun, one process per GPU)
every rank gates its own batch of T tokens (token shards, no collective on the
data path: weak scaling); time is the max over ranks.

``--impl reference`` times the CPU oracle (the fp64 definition, as it stands)
on this host's cores, on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import datetime
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

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "fused top-k gating tokens/s"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NVML_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
                0x2: "applications_clocks_setting", 0x10: "sync_boost"}
PROFILE_DIR = os.path.join(ROOT, "profiles")


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[1])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="train", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workspace", action="store_true",
                    help="time tk_gating_fused_topk (no workspace) instead of tk_gating_fused_topk_ws, whose many-token "
                         "launches split their last round between CTA pairs")
    ap.add_argument("--no-workload-summary", action="store_true",
                    help="skip the per-workload table (every router workload, GPU and oracle, one GPU only)")
    ap.add_argument("--tokens", type=int, default=None, help="override T of the workload (profiling cases)")
    ap.add_argument("--precision", default="bf16", choices=("bf16", "fp8"),
                    help="bf16 (default) or FP8 E4M3 inputs with per-token / per-expert scales")
    ap.add_argument("--op", default="gating", choices=("gating", "route", "gating_route", "ep"),
                    help="gating (default); route: routing metadata of the workload's T x k ids; "
                         "gating_route: both, chained on the device; ep: expert-parallel dispatch and combine "
                         "of the workload's tokens (one rank)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (earlier measurement on this pool)"


def of_peaks(peak_src: str) -> str:
    """How a roofline fraction names its denominator: measured on this machine, or the fallback."""
    return "of measured" if peak_src.startswith("measured") else "of fallback"


def workload_desc(wl):
    extra = ""
    if wl.kind == "skew":
        extra = f", +3u shared direction, dominant {list(wl.dominant)}, duplicated pairs {list(wl.duplicate_pairs)}"
    return (f"{wl.name}: T={wl.T} H={wl.H} E={wl.E} k={wl.k}; synthetic bf16 hidden ~N(0,1), "
            f"gate ~N(0,1/H), seed {wl.seed}{extra}")


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def time_oracle(wl, seconds: float):
    """Oracle tokens/s on a bounded row sample of `wl` (rows from the start):
    doubles the sample until one timed run takes at least `seconds`."""
    import oracle
    orc = oracle.load()
    w_bits = wl.gate_weight()
    rows = min(wl.T, 64)
    while True:
        x = wl.hidden_rows(0, rows)
        t0 = time.perf_counter()
        orc.gating(x, w_bits, wl.k)
        dt = time.perf_counter() - t0
        if dt >= seconds or rows == wl.T:
            return rows / dt, rows, dt, orc.max_threads()
        rows = int(min(wl.T, max(rows * 2, rows * 1.2 * seconds / max(dt, 1e-6))))


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    orc = oracle.load()
    w_bits = wl.gate_weight()
    total_steps = args.steps + args.warmup
    per_step_s = max(0.05, min(2.0, 150.0 / max(total_steps, 1)))
    probe = min(wl.T, 32)
    t0 = time.perf_counter()
    orc.gating(wl.hidden_rows(0, probe), w_bits, wl.k)
    rate = probe / max(time.perf_counter() - t0, 1e-6)
    rows = int(min(wl.T, max(1, rate * per_step_s)))
    x = wl.hidden_rows(0, rows)
    for _ in range(args.warmup):
        orc.gating(x, w_bits, wl.k)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.gating(x, w_bits, wl.k)
    dt = time.perf_counter() - t0
    value = rows * args.steps / dt
    sample = f"first {rows} of {wl.T} tokens per step (fp64 oracle, full sort), same gate"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(wl), "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k,
                   "tokens_per_step": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.max_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    def __init__(self, local_rank: int, period_s: float = 0.0005):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            cvd = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [s.strip() for s in cvd.split(",") if s.strip()]
            if ids and local_rank < len(ids):
                tok = ids[local_rank]
                h = (pynvml.nvmlDeviceGetHandleByIndex(int(tok)) if tok.isdigit()
                     else pynvml.nvmlDeviceGetHandleByUUID(tok))
            else:
                h = pynvml.nvmlDeviceGetHandleByIndex(local_rank)
            self._nvml, self._h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception as e:  # no NVML: report clocks as unavailable
            self._nvml = None
            self.error = repr(e)

    def _run(self):
        # only the SM clock and the event reasons every period (cheap queries);
        # the power reading is slower and is taken every 8th sample
        p, h = self._nvml, self._h
        power = None
        i = 0
        self.query_s = []
        while not self._stop.is_set():
            t0 = time.perf_counter()
            try:
                sm = p.nvmlDeviceGetClockInfo(h, p.NVML_CLOCK_SM)
                reasons = self._reasons(h)
                if i % 8 == 0:
                    power = p.nvmlDeviceGetPowerUsage(h) / 1000.0
                if self._recording:
                    self.samples.append((sm, reasons, power))
            except Exception as e:
                self.error = repr(e)
            self.query_s.append(time.perf_counter() - t0)
            i += 1
            self._ready.set()
            self._stop.wait(self.period)

    def __enter__(self):
        # the thread's first NVML queries (which may take milliseconds) run before
        # the timed region; only samples taken inside it are kept
        self._recording = False
        self._ready = threading.Event()
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
            self._ready.wait(1.0)
        self._recording = True
        return self

    def __exit__(self, *exc):
        self._recording = False
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": f"NVML unavailable: {self.error}"}
        # the sampler runs only while the timed launches run, so every sample is
        # under load (NVML's utilisation counter lags and is not used to filter)
        reasons = set()
        for s in self.samples:
            for bit, name in NVML_REASONS.items():
                if s[1] & bit and name != "gpu_idle":
                    reasons.add(name)
        return {
            "sm_mhz": statistics.median([s[0] for s in self.samples]) if self.samples else None,
            "sm_mhz_min": min([s[0] for s in self.samples]) if self.samples else None,
            "sm_max_mhz": self.max_mhz,
            "reasons": sorted(reasons),
            "samples": len(self.samples),
            "power_w_max": max([s[2] for s in self.samples if s[2] is not None], default=None),
            "source": "NVML (same counters as nvidia-smi), sampled every %.1f ms during the timed region"
                      % (self.period * 1e3),
            "nvml_query_ms_median": (statistics.median(self.query_s[1:]) * 1e3
                                     if len(getattr(self, "query_s", [])) > 1 else None),
        }


def wait_releasing_gil(event) -> None:
    """Wait for `event` by polling with short sleeps, so that the clock sampler's
    thread gets the interpreter while the timed launches run (a blocking
    synchronize may hold it); the caller still synchronizes afterwards."""
    while not event.query():
        time.sleep(0.0002)


# ---------------------------------------------------------------------------
def kernel_source_digest() -> str:
    from moe_router_gating_b200 import build as tkbuild
    return tkbuild.gating_kernel_digest()


def profiled_traffic(wl, digest: str, suffix: str = ""):
    """dram read+write bytes per launch from a committed ncu summary, if it was
    taken on the current kernel sources (same digest); else None."""
    path = os.path.join(PROFILE_DIR, f"traffic_{wl.name}{suffix}.txt")
    if not os.path.exists(path):
        return None, None
    vals = {}
    with open(path) as f:
        for line in f:
            if "=" in line and not line.lstrip().startswith("#"):
                k, v = line.split("=", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_digest") != digest:
        return None, f"{os.path.basename(path)} was taken on other kernel sources"
    return float(vals["dram_bytes_per_launch"]), os.path.basename(path)


# ---------------------------------------------------------------------------
# multi-rank host logic (one process per GPU; also exercised by CPU gloo tests)
# ---------------------------------------------------------------------------
def rank_workload(wl, rank: int):
    """Each rank gates its own batch of T tokens: the same shapes, another seed."""
    return workloads.RouterWorkload(wl.name, wl.T, wl.H, wl.E, wl.k, wl.kind, wl.seed + rank,
                                    wl.dominant, wl.duplicate_pairs)


def max_over_ranks(value_ms: float, device, world: int) -> float:
    """The slowest rank's time (all ranks take part in the reduction)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, steps: int, elapsed_max_ms: float) -> float:
    """Whole-job throughput: the tokens all ranks gated, over the slowest rank's time."""
    return world * tokens_per_rank * steps / (elapsed_max_ms / 1e3)


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    import moe_router_gating_b200 as tk

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- inputs: seeded host arrays, each rank gates its own token shard ----
    rank_wl = rank_workload(wl, rank)
    fp8 = args.precision == "fp8"
    scores = torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    if fp8:
        xq, xs, wq, ws = workloads.fp8_inputs(rank_wl)
        x_host = torch.from_numpy(xq)
        xs_host = torch.from_numpy(xs)
        x, xsd = x_host.to(dev), xs_host.to(dev)
        wqd, wsd = torch.from_numpy(wq).to(dev), torch.from_numpy(ws).to(dev)
        hidden_bytes = wl.T * wl.H + 4 * wl.T

        work = None if args.no_workspace else tk.gating_workspace(wl.T, wl.H, wl.E, wl.k, dev, fp8=True)

        def gate(xx):
            return lambda: tk.fused_topk_gating_fp8(xx, xsd, wqd, wsd, wl.k, scores=scores, ids=ids, stream=stream,
                                                    workspace=work)
    else:
        x_host = workloads.to_torch_bf16(rank_wl.hidden())
        w = workloads.to_torch_bf16(rank_wl.gate_weight()).to(dev)
        x = x_host.to(dev)
        hidden_bytes = wl.T * wl.H * 2

        work = None if args.no_workspace else tk.gating_workspace(wl.T, wl.H, wl.E, wl.k, dev)

        def gate(xx):
            return lambda: tk.fused_topk_gating(xx, w, wl.k, scores=scores, ids=ids, stream=stream, workspace=work)
    big = hidden_bytes > L2_BYTES
    # 16 MB up to L2: back-to-back launches over rotating hidden buffers that together
    # exceed twice L2 (each launch reads a hidden tensor evicted since its last use)
    rotate = not big and hidden_bytes >= 16 * 1024 * 1024
    n_buf = max(4, -(-2 * L2_BYTES // hidden_bytes) + 1) if rotate else 1
    xs_dev = [x] + [x.clone() for _ in range(n_buf - 1)]
    steps_of = [gate(xx) for xx in xs_dev]
    step_count = [0]

    def step():
        steps_of[step_count[0] % n_buf]()
        step_count[0] += 1
    flush = None if big or rotate else torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    tk.device_error(clear=True)

    sampler = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize(dev)
    tk.clock_counters(clear=True)
    with sampler:
        if big or rotate:
            # inputs larger than L2 (or rotating buffers): back-to-back launches between two events
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            for _ in range(args.steps):
                step()
            ev1.record(stream)
            wait_releasing_gil(ev1)
            torch.cuda.synchronize(dev)
            elapsed_ms = ev0.elapsed_time(ev1)
            launch_ms = elapsed_ms / args.steps
        else:
            # small inputs: flush L2 (write 2x L2) between steps, time each launch alone
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for a, b in evs:
                flush.zero_()
                a.record(stream)
                step()
                b.record(stream)
            wait_releasing_gil(evs[-1][1])
            torch.cuda.synchronize(dev)
            per = [a.elapsed_time(b) for a, b in evs]
            elapsed_ms = sum(per)
            launch_ms = elapsed_ms / args.steps
    torch.cuda.synchronize(dev)
    kernel_clock = tk.clock_counters(clear=True)  # SM clock of the timed launches themselves
    barrier()
    err = tk.device_error(clear=True)
    if err:
        raise SystemExit(f"device error word {err:#x}: a kernel wait expired during the timed region")

    elapsed_max_ms = max_over_ranks(elapsed_ms, dev, world)
    ms_per_step = elapsed_max_ms / args.steps
    value = job_tokens_per_s(world, wl.T, args.steps, elapsed_max_ms)

    # ---- end to end through the host-buffer C-ABI call (pinned host memory) ----
    x_pinned = x_host.pin_memory()
    s_host = torch.empty((wl.T, wl.k), dtype=torch.float32).pin_memory()
    i_host = torch.empty((wl.T, wl.k), dtype=torch.int32).pin_memory()
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    if fp8:
        xs_pinned = xs_host.pin_memory()

        def e2e_step():  # host buffers in and out around the public FP8 call
            x.copy_(x_pinned, non_blocking=True)
            xsd.copy_(xs_pinned, non_blocking=True)
            tk.fused_topk_gating_fp8(x, xsd, wqd, wsd, wl.k, scores=scores, ids=ids, stream=stream)
            s_host.copy_(scores, non_blocking=True)
            i_host.copy_(ids, non_blocking=True)
    else:
        def e2e_step():
            tk.fused_topk_gating_host(x_pinned, w, wl.k, s_host, i_host, x, scores, ids, stream=stream)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_value = job_tokens_per_s(world, wl.T, e2e_steps, max_over_ranks(e0.elapsed_time(e1), dev, world))

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    # ---- roofline of the (only) kernel ----
    peaks, peak_src = load_peaks()
    roofline = roofline_of(wl, launch_ms, fp8, peaks, peak_src)
    digest = kernel_source_digest()
    traffic, traffic_src = profiled_traffic(wl, digest, "_fp8" if fp8 else "")
    roofline["traffic"] = traffic
    roofline.update({"traffic_source": traffic_src, "kernel_source_digest": digest})

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    plan_h = wl.H // 2 if fp8 else wl.H
    plan = tk.make_plan(wl.T, plan_h, wl.E, wl.k, sms) if args.no_workspace else \
        tk.make_plan_ws(wl.T, plan_h, wl.E, wl.k, sms)[0]

    cpu = None
    if not args.no_cpu_baseline and world == 1 and not fp8:
        v, rows, dt, cores = time_oracle(wl, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"first {rows} of {wl.T} tokens ({dt:.1f} s, fp64 oracle with full sort, all host threads)"}

    per_workload = None
    if world == 1 and not fp8 and not args.no_workload_summary and args.tokens is None:
        per_workload = per_workload_summary(dev, peaks, peak_src, min(args.cpu_seconds, 2.0),
                                            not args.no_cpu_baseline)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
        "config": {
            "workload": workload_desc(wl), "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k,
            "tokens_per_rank_per_step": wl.T,
            "arithmetic": ("e4m3 x e4m3 products, fp32 accumulate (tcgen05 kind::f8f6f4), per-expert and per-token "
                           "scales in fp32, fp32 top-k and softmax" if fp8 else
                           "bf16 x bf16 products, fp32 accumulate (tcgen05), fp32 top-k and softmax"),
            "precision": args.precision,
            "l2": ("inputs larger than L2: hidden is %.0f MB per step (gate %.2f MB stays L2-resident by design)"
                   % (hidden_bytes / 1e6, wl.H * wl.E * 2 / 1e6)) if big else
                  ("back-to-back launches over %d hidden buffers (%.0f MB together, more than twice L2); the gate "
                   "stays L2-resident by design" % (n_buf, n_buf * hidden_bytes / 1e6)) if rotate else
                  "L2 flushed (256 MB write) before every timed launch; each launch timed alone",
            "parallelism": "single GPU" if world == 1 else f"{world} ranks, independent token shards, no collective",
            "launch": plan,
            "entry": "tk_gating_fused_topk" if args.no_workspace else "tk_gating_fused_topk_ws",
        },
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": hidden_bytes,
                "d2h_bytes_per_step": wl.T * wl.k * 8,
                "path": ("pinned host hidden_q + scales -> device, tk_gating_fused_topk_fp8, scores+ids -> pinned host"
                         if fp8 else
                         "tk_gating_fused_topk_host: pinned host hidden -> device, kernel, scores+ids -> pinned host")},
        "gpu_launches": args.steps,
        "clocks": clocks_summary(sampler, kernel_clock, launch_ms),
    }
    if per_workload is not None:
        line["workloads"] = per_workload
    print(json.dumps(line), flush=True)
    return 0


def roofline_of(wl, launch_ms: float, fp8: bool, peaks: dict, peak_src: str) -> dict:
    """Roofline of one launch: the binding term at the burst peaks, and the
    fraction of the roofline at both the burst and the sustained tensor peak
    (neither is picked by the length of the run)."""
    bytes_alg = wl.algorithmic_bytes()
    flops = wl.flops()
    tc_factor = 1.0
    if fp8:  # 1-byte operands plus the scales; the FP8 tensor peak is twice the bf16 one (nominal ratio)
        bytes_alg = wl.T * wl.H + wl.E * wl.H + 4 * (wl.T + wl.E) + 8 * wl.T * wl.k
        tc_factor = 2.0
    t_s = launch_ms / 1e3
    hbm_ach = bytes_alg / t_s / 1e9
    tc_ach = flops / t_s / 1e12
    tc_burst = tc_factor * peaks["bf16_tflops"]
    tc_sust = tc_factor * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    t_hbm = bytes_alg / (peaks["hbm_gbs"] * 1e9)
    t_tc_burst = flops / (tc_burst * 1e12)
    t_tc_sust = flops / (tc_sust * 1e12)
    hbm = {"bound": "hbm", "achieved": hbm_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
           "frac": hbm_ach / peaks["hbm_gbs"]}
    tc = {"bound": "tensor", "achieved": tc_ach, "peak": tc_burst, "unit": "TFLOP/s", "frac": tc_ach / tc_burst}
    primary, secondary = (hbm, tc) if t_hbm >= t_tc_burst else (tc, hbm)
    roof = dict(primary)
    roof.update({
        "peak_source": (f"{peak_src}; HBM = copy GB/s ({of_peaks(peak_src)}); tensor = cuBLAS bf16 burst "
                        f"TFLOP/s ({of_peaks(peak_src)}){'; x2 for FP8 (nominal FP8/bf16 ratio)' if fp8 else ''}"),
        "roofline_frac": max(t_hbm, t_tc_burst) / t_s,
        "roofline_frac_sustained": max(t_hbm, t_tc_sust) / t_s,
        "tensor_frac_sustained": tc_ach / tc_sust,
        "roofline_us": {"hbm": t_hbm * 1e6, "tensor_burst": t_tc_burst * 1e6, "tensor_sustained": t_tc_sust * 1e6},
        "algorithmic_bytes_per_launch": bytes_alg, "flops_per_launch": flops, "launch_ms": launch_ms,
        "secondary": {k: secondary[k] for k in ("bound", "achieved", "peak", "unit", "frac")},
    })
    return roof


def clocks_summary(sampler, kernel_clock: dict, launch_ms: float) -> dict:
    """NVML samples of the timed region, plus the SM clock the launches measured
    on themselves (first CTA: clock64 cycles over globaltimer ns)."""
    c = sampler.summary()
    ghz = kernel_clock.get("sm_ghz")
    c["sm_mhz_in_kernel"] = ghz * 1e3 if ghz else None
    c["in_kernel_launches"] = kernel_clock.get("launches")
    c["cycles_per_launch"] = ghz * 1e9 * launch_ms / 1e3 if ghz else None
    c["in_kernel_source"] = ("first CTA of every timed launch: SM clock64 cycles / globaltimer ns, "
                             "summed over the launches (tk_gating_clock_counters)")
    return c


# The synthetic router workloads the gating is specified on, each measured in
# the same run as the headline (one GPU): tokens/s, us per call and the roofline
# fraction, next to the CPU oracle on a bounded sample of the same workload.
SUMMARY_WORKLOADS = ("tiny", "deepseek", "skew", "train", "decode_T1", "decode_T8", "decode_T32", "decode_T128",
                     "decode_T256")


def time_calls(step, stream, steps: int, flush) -> float:
    """Mean ms per call: each call timed alone with CUDA events after an L2 flush
    (flush is None for inputs larger than L2: back-to-back calls between two events)."""
    import torch
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if flush is None:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / steps


def oracle_single_thread_rate(wl, seconds: float):
    """The oracle's tokens/s with one OpenMP thread (the same code, one core)."""
    import ctypes
    gomp = ctypes.CDLL("libgomp.so.1")
    before = gomp.omp_get_max_threads()
    gomp.omp_set_num_threads(1)
    try:
        v, rows, dt, _ = time_oracle(wl, seconds)
    finally:
        gomp.omp_set_num_threads(before)
    return v, rows, dt


def time_rotating(steps_of, stream, steps: int) -> float:
    """Mean ms per call of back-to-back calls that cycle through distinct input
    buffers (steps_of[i] gates buffer i): each call reads a hidden tensor that
    the calls since its last use have evicted from L2."""
    import torch
    for st in steps_of:
        st()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        steps_of[i % len(steps_of)]()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def per_workload_summary(dev, peaks, peak_src, cpu_seconds: float, with_cpu: bool) -> dict:
    """Every router workload on one GPU.  Timing: inputs larger than L2 back to
    back; inputs of 16 MB up to L2 back to back over rotating hidden buffers
    (together more than twice L2; the gate stays L2-resident by design);
    smaller ones one call at a time after an L2 flush.  Each entry also gives
    the one-call-after-a-flush time (which carries the ~5 us launch latency
    after the flush kernel) and the kernel's own span measured in the kernel."""
    import torch

    import moe_router_gating_b200 as tk
    out = {}
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    for name in SUMMARY_WORKLOADS:
        wl = workloads.WORKLOADS[name]
        hidden_bytes = wl.T * wl.H * 2
        x = workloads.to_torch_bf16(wl.hidden()).to(dev)
        w = workloads.to_torch_bf16(wl.gate_weight()).to(dev)
        s = torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev)
        i = torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev)
        big = hidden_bytes > L2_BYTES
        rotate = not big and hidden_bytes >= 16 * 1024 * 1024

        work = tk.gating_workspace(wl.T, wl.H, wl.E, wl.k, dev)

        def gate(xx):
            return lambda: tk.fused_topk_gating(xx, w, wl.k, scores=s, ids=i, stream=stream, workspace=work)
        flushed_ms = None
        if not big:
            tk.clock_counters(clear=True)
            flushed_ms = time_calls(gate(x), stream, 200, flush)
        clk = tk.clock_counters(clear=True)
        if big:
            ms = time_calls(gate(x), stream, 20, None)
            clk = tk.clock_counters(clear=True)
            timing = "back-to-back calls, inputs larger than L2"
        elif rotate:
            n = max(4, -(-2 * L2_BYTES // hidden_bytes) + 1)
            xs = [x] + [x.clone() for _ in range(n - 1)]
            ms = time_rotating([gate(xx) for xx in xs], stream, 20 * n)
            clk = tk.clock_counters(clear=True)
            timing = (f"back-to-back calls over {n} hidden buffers ({n * hidden_bytes / 1e6:.0f} MB, more than "
                      "twice L2); the gate stays L2-resident")
            del xs
        else:
            ms = flushed_ms
            timing = "each call alone after an L2 flush (256 MB write), mean of 200"
        roof = roofline_of(wl, ms, False, peaks, peak_src)
        launches = clk["launches"] or 1
        entry = {"T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "us_per_call": ms * 1e3,
                 "tokens_per_s": wl.T / (ms / 1e3), "timing": timing,
                 "us_per_call_after_flush": flushed_ms * 1e3 if flushed_ms is not None else None,
                 "kernel_span_us_in_kernel": clk["elapsed_ns"] / launches / 1e3 if clk["launches"] else None,
                 "roofline": {"bound": roof["bound"], "frac": roof["frac"], "roofline_frac": roof["roofline_frac"],
                              "roofline_frac_sustained": roof["roofline_frac_sustained"],
                              "roofline_us": roof["roofline_us"]},
                 "sm_mhz_in_kernel": clk["sm_ghz"] * 1e3 if clk["sm_ghz"] else None,
                 "plan": {k: v for k, v in tk.make_plan_ws(wl.T, wl.H, wl.E, wl.k,
                                                           torch.cuda.get_device_properties(dev).multi_processor_count)[0]
                          .items() if k in ("variant", "cluster", "grid", "num_tiles", "num_half_tiles",
                                            "num_split_tiles")},
                 "entry": "tk_gating_fused_topk_ws"}
        if err := tk.device_error(clear=True):
            raise SystemExit(f"device error word {err:#x} during the {name} summary")
        if with_cpu:
            v, rows, dt, cores = time_oracle(wl, cpu_seconds)
            entry["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                     "sample": f"first {rows} of {wl.T} tokens ({dt:.2f} s)"}
            if name == "deepseek":
                v1, rows1, dt1 = oracle_single_thread_rate(wl, cpu_seconds)
                entry["cpu_baseline_1thread"] = {"value": v1, "unit": UNIT, "cores": 1, "kind": "oracle",
                                                 "sample": f"first {rows1} of {wl.T} tokens ({dt1:.2f} s)"}
        out[name] = entry
        del x, w, s, i
    return out


# ---------------------------------------------------------------------------
# routing metadata (--op route / gating_route), one GPU
# ---------------------------------------------------------------------------
ROUTE_METRIC = "routing metadata tokens/s"
CHAIN_METRIC = "gating + routing tokens/s"


def route_bytes(T: int, k: int, E: int) -> int:
    """ids read once; sorted_slots, slot_pos and offsets written once."""
    return 12 * T * k + 4 * (E + 1)


def time_route_oracle(T, k, E, seconds: float):
    import oracle
    orc = oracle.load()
    ids = workloads.expert_ids(T, k, E, seed=0)
    reps, dt = 0, 0.0
    t0 = time.perf_counter()
    while dt < seconds:
        orc.route(ids, E)
        reps += 1
        dt = time.perf_counter() - t0
    return T * reps / dt, reps, dt


def run_route_ours(args, wl):
    import torch

    import moe_router_gating_b200 as tk
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--op route runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, k, E = wl.T, wl.k, wl.E
    chain = args.op == "gating_route"
    stream = torch.cuda.current_stream(dev)
    ids_host = torch.from_numpy(workloads.expert_ids(T, k, E, seed=0))
    ids = ids_host.to(dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_slots = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    if chain:
        x = workloads.to_torch_bf16(wl.hidden()).to(dev)
        w = workloads.to_torch_bf16(wl.gate_weight()).to(dev)
        scores = torch.empty((T, k), dtype=torch.float32, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    if chain:
        # gating and routing in one call: the gating kernel counts the assignments
        # per expert, the placing kernel follows (tk_gating_fused_topk_route)
        ws = tk.route_workspace(T, k, E, dev)
        H = x.shape[1]

        def step():
            st = tk.fused_topk_gating_route_ptr(x.data_ptr(), w.data_ptr(), T, H, E, k, scores.data_ptr(),
                                                ids.data_ptr(), offsets.data_ptr(), sorted_slots.data_ptr(),
                                                slot_pos.data_ptr(), ws.data_ptr(), ws.numel() * 4,
                                                stream.cuda_stream)
            if st != tk.TK_OK:
                raise SystemExit(f"tk_gating_fused_topk_route: {tk.status_string(st)}")
    else:
        def step():
            tk.route(ids, E, offsets, sorted_slots, slot_pos, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    tk.device_error(clear=True)
    sampler = ClockSampler(0)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with sampler:
        for a, b in evs:
            flush.zero_()  # ids (and the gate) would otherwise stay in L2 between steps
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize(dev)
    per = [a.elapsed_time(b) for a, b in evs]
    if tk.device_error(clear=True):
        raise SystemExit("a kernel wait expired during the timed region")
    elapsed_ms = sum(per)
    ms_per_step = elapsed_ms / args.steps
    value = T * args.steps / (elapsed_ms / 1e3)
    gating_alone_ms = chained_ms = None
    if chain:
        # timed the same way in the same run: the gating call alone (the routing's
        # added cost), and the two separate calls (gating, then tk_gating_route,
        # which counts the ids in a launch of its own)
        def timed(fn):
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for a, b in evs:
                flush.zero_()
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize(dev)
            return sum(a.elapsed_time(b) for a, b in evs) / args.steps

        gating_alone_ms = timed(lambda: tk.fused_topk_gating(x, w, k, scores=scores, ids=ids, stream=stream))
        # the separate calls through the no-allocation routing entry point (the same
        # kernels as tk_gating_route, without its stream-ordered workspace allocation)
        chained_ms = timed(lambda: (tk.fused_topk_gating(x, w, k, scores=scores, ids=ids, stream=stream),
                                    tk.route_static_ptr(ids.data_ptr(), T, k, E, offsets.data_ptr(),
                                                        sorted_slots.data_ptr(), slot_pos.data_ptr(),
                                                        stream.cuda_stream)))

    # end to end: pinned host ids -> device, route, the three outputs -> pinned host
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    ids_pinned = ids_host.pin_memory()
    outs_host = [torch.empty(t.shape, dtype=torch.int32).pin_memory() for t in (offsets, sorted_slots, slot_pos)]

    def e2e_step():
        ids.copy_(ids_pinned, non_blocking=True)
        tk.route(ids, E, offsets, sorted_slots, slot_pos, stream=stream)
        for h, d in zip(outs_host, (offsets, sorted_slots, slot_pos)):
            h.copy_(d, non_blocking=True)

    e2e_value = None
    if not chain:
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_value = T * e2e_steps / (e0.elapsed_time(e1) / 1e3)

    peaks, peak_src = load_peaks()
    bytes_alg = route_bytes(T, k, E)
    plan = tk.route_plan(T, k, E, torch.cuda.get_device_properties(dev).multi_processor_count)
    line = {
        "metric": CHAIN_METRIC if chain else ROUTE_METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int32" if not chain else "bf16", "data": "synthetic",
        "config": {"workload": (workload_desc(wl) if chain else
                                f"route of {wl.name}-shaped ids: T={T} k={k} E={E}, uniform seeded ids, "
                                "k distinct per token"),
                   "T": T, "k": k, "E": E,
                   "l2": "L2 flushed (256 MB write) before every timed step; each step timed alone",
                   "launch": plan},
        "gpu_launches": args.steps * 2,  # gating + placing kernel, or counting + placing kernel
        "clocks": sampler.summary(),
    }
    if chain:
        line["path"] = "tk_gating_fused_topk_route (counts taken in the gating epilogue)"
        line["gating_alone_ms_per_step"] = gating_alone_ms
        line["routing_added_us"] = (ms_per_step - gating_alone_ms) * 1e3
        line["separate_calls_ms_per_step"] = chained_ms
        line["separate_calls_routing_added_us"] = (chained_ms - gating_alone_ms) * 1e3
        line["separate_calls_path"] = ("tk_gating_fused_topk, then tk_gating_route_static (count kernel + "
                                       "placing kernel, no allocation)")
    if not chain:
        ach = bytes_alg / (ms_per_step / 1e3) / 1e9
        line["roofline"] = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": ach / peaks["hbm_gbs"], "traffic": None,
                            "peak_source": f"{peak_src}; copy GB/s ({of_peaks(peak_src)})",
                            "algorithmic_bytes_per_step": bytes_alg,
                            "note": "two launches per step (count, then scatter); time of the pair"}
        line["e2e"] = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": 4 * T * k,
                       "d2h_bytes_per_step": 4 * (E + 1) + 8 * T * k,
                       "path": "pinned host ids -> device, tk_gating_route, three outputs -> pinned host"}
        if not args.no_cpu_baseline:
            v, reps, dt = time_route_oracle(T, k, E, min(args.cpu_seconds, 5.0))
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                                    "sample": f"whole workload, {reps} calls in {dt:.1f} s (single-thread C)"}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# expert-parallel dispatch and combine (--op ep), one GPU, one rank
# ---------------------------------------------------------------------------
EP_METRIC = "expert-parallel dispatch + combine tokens/s"


def run_ep_ours(args, wl):
    """Dispatch copies every placed assignment's token row to its expert row;
    combine sums each token's k expert rows.  One rank, so every row stays in
    this GPU's memory; each kernel is timed on its own (CUDA events, inputs
    larger than L2 at the 4096-token shape: T*k rows of 14 KB = 470 MB)."""
    import torch

    import moe_router_gating_b200 as tk
    from moe_router_gating_b200 import ep
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, H, E, k = wl.T, wl.H, wl.E, wl.k
    stream = torch.cuda.current_stream(dev)
    x = workloads.to_torch_bf16(wl.hidden()).to(dev)
    ids = torch.from_numpy(workloads.expert_ids(T, k, E, seed=0, kind="skew")).to(dev)
    scores = torch.rand((T, k), dtype=torch.float32, device=dev)
    g = ep.ExpertParallelGroup(E, H, capacity=T * k, device=dev)
    offsets, sorted_slots, slot_pos = tk.route(ids, E)
    rows, out_rows, recv_offsets = ep.rows_table(offsets.view(1, E + 1), 0, g.bases, g.out_bases, H)
    g.output.copy_(g.recv)  # experts = identity for the timing
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)

    def dispatch():
        ep.dispatch_rows(x, ids, offsets, slot_pos, rows, E, stream)

    def combine():
        ep.combine_rows(out_rows, ids, offsets, slot_pos, scores, out, E, stream)

    def timed(fn, steps):
        for _ in range(max(args.warmup, 3)):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / steps

    tk.device_error(clear=True)
    sampler = ClockSampler(0)
    with sampler:
        t_d = timed(dispatch, args.steps)
        t_c = timed(combine, args.steps)
    if tk.device_error(clear=True):
        raise SystemExit("an expert-parallel kernel reported a bad row address")
    placed = T * k
    d_bytes = 2 * H * T + (2 * H) * placed    # each token row read once, each placed row written once
    c_bytes = (2 * H) * placed + 2 * H * T + 12 * T * k   # k rows read per token, one row written, metadata
    peaks, peak_src = load_peaks()
    ms = t_d + t_c
    line = {
        "metric": EP_METRIC, "value": T / (ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{wl.name}-shaped tokens: T={T} H={H} E={E} k={k}, skewed seeded ids, one rank",
                   "l2": "dispatch writes and combine reads 470 MB of expert rows per step (more than L2)"},
        "roofline": {"bound": "hbm", "dispatch_us": t_d * 1e3, "combine_us": t_c * 1e3,
                     "dispatch_gbs": d_bytes / (t_d / 1e3) / 1e9, "combine_gbs": c_bytes / (t_c / 1e3) / 1e9,
                     "dispatch_frac": d_bytes / (t_d / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "combine_frac": c_bytes / (t_c / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "peak_source": f"{peak_src}; copy GB/s ({of_peaks(peak_src)})",
                     "algorithmic_bytes": {"dispatch": d_bytes, "combine": c_bytes}},
        "gpu_launches": args.steps * 2,
        "clocks": sampler.summary(),
        "note": "one rank: every row stays local; across GPUs the same stores and loads go to peer memory "
                "(not measured: one GPU per call on this pool)",
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens is not None:
        wl = wl.with_T(args.tokens)
    if args.op != "gating":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers --op gating only"}))
            return 0
        if args.op == "ep":
            return run_ep_ours(args, wl)
        return run_route_ours(args, wl)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
