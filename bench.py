#!/usr/bin/env python
"""Throughput of the decode-time MoE layer on B200: µs/layer, tokens/s and HBM GB/s.

One step = one call of the whole layer (router GEMV, top-k routing, grouping by expert,
gate+up+SwiGLU, down projection with the weighted blend and shared expert) on m rows of a seeded
synthetic layer. Steps rotate over R replicas of the layer's weights (same values, separate
device memory) and over the 64-row activation pool, so the weights touched between two uses of
a replica exceed 4x the L2 cache: every timed call streams its weights from HBM.

Headline workload (the largest shape of the metric "µs and tokens/s at m = 1..64"): the
Llama-4-Scout-shaped layer (hidden 5120, 16 experts, top-1 on raw logits with the weight before
the FFN, moe_intermediate 8192, shared expert 8192, bf16 weights) at m = 64. The same JSON line
carries a `sweep` list: every published shape at each of its row counts, each timed as the
median of 5 windows.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--m M] [--no-sweep]
  python bench.py --impl reference ...     # the float64 CPU oracle on the host cores

With N > 1 (torchrun) every rank runs an independent replica of the workload on its own GPU
(no collective on the data path; the layer does not shard) and rank 0 prints the whole-job line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "MoE decode layer µs and tokens/s at m=1..64; achieved HBM GB/s vs B200 peak"
HEADLINE = ("llama4_scout", 64)
SWEEP_CONFIGS = ("qwen3_30b_a3b", "lfm2_8b_a1b", "qwen3_6_35b_a3b", "llama4_scout",
                 "qwen3_30b_a3b_mxfp4", "qwen3_30b_a3b_fp8")

# DRAM bytes per call (dram__bytes_read.sum + dram__bytes_write.sum summed over the call's
# launches, one ncu capture of the current kernels; the summaries are in profiles/). Keyed by
# (workload config name, m); entries are removed whenever the kernels they measured change.
# DRAM bytes (read + write) per launch of the layer's kernel, from a single-pass ncu capture of
# the same workload (profiles/tc_fused_kernel_traffic_llama4_scout_m64.md); retaken whenever the
# kernel changes.
PROFILED_TRAFFIC: dict = {("llama4_scout", 64): 4.03e9 + 5.9e6}
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
WINDOWS = 5


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", default=HEADLINE[0])
    ap.add_argument("--m", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cold-steps", type=int, default=30,
                    help="calls timed one by one after an L2 flush (0: skip)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="time the headline workload only")
    ap.add_argument("--sweep-steps", type=int, default=64,
                    help="calls per timed window of a sweep entry (rounded up to the replicas)")
    ap.add_argument("--path", choices=("auto", "chain"), default="auto",
                    help="launch path: the automatic choice, or the multi-kernel path at every m")
    ap.add_argument("--replicas", type=int, default=None,
                    help="weight replicas (default: enough for 4x L2 between reuses)")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def touched_bytes(cfg, active_count: int) -> int:
    """Algorithmic bytes of one call: router + distinct selected experts + shared expert."""
    from mixture_experts_decode_gemv_b200.synthetic import weight_bytes_per_expert
    xb = 2 if cfg.x_dtype == "bf16" else 4
    n = cfg.num_experts * cfg.hidden * xb
    n += active_count * weight_bytes_per_expert(cfg)
    if cfg.has_shared:
        n += weight_bytes_per_expert(cfg, inter=cfg.shared_inter)
        if cfg.shared_kind == "sigmoid_gate":
            n += cfg.hidden * xb
    return n


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.proc = None
        if enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "100", "-i", str(gpu_index)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (OSError, FileNotFoundError):
                self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def max_over_ranks(v: float, ws: int, device: str = "cuda") -> float:
    """The largest of the ranks' values (a rank's timed milliseconds): the job's time."""
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def workload_name(cfg, m):
    return (f"{cfg.name} m={m}: hidden {cfg.hidden}, {cfg.num_experts} experts, top-{cfg.top_k}, "
            f"moe_intermediate {cfg.moe_inter}"
            + (f", shared {cfg.shared_inter} ({cfg.shared_kind})" if cfg.has_shared else "")
            + f", {cfg.fmt} weights, {cfg.routing} routing"
            + (", weight before the FFN" if cfg.weight_before_ffn else ""))


def config_dict(cfg, m, wsz):
    """The `config` of the JSON line; identical for both arms of the same workload."""
    return {"workload": workload_name(cfg, m), "m": m, "weights": cfg.fmt,
            "l2_policy": "inputs larger than L2: weight replicas and activation batches rotate, "
                         ">= 4x L2 between reuses of a replica",
            "parallelism": f"replicas x{wsz}"}


def oracle_rows_per_second(lay, m, seconds, chunk=8):
    """The float64 oracle, as it stands, on a bounded sample of the workload: rows of the m-row
    batches evaluated `chunk` at a time (each call routes its whole batch and evaluates the rows
    of the chunk) until `seconds` have passed. Returns (rows/s, rows, calls, elapsed)."""
    from mixture_experts_decode_gemv_b200.synthetic import POOL_ROWS
    from oracle import moe_ref as ref
    olay = ref.OracleLayer(lay)
    nx = max(1, POOL_ROWS // m)
    per_batch = max(1, math.ceil(m / chunk))
    rows = calls = 0
    t0 = time.perf_counter()
    while True:
        b, lo = calls // per_batch, (calls % per_batch) * chunk
        sel = list(range(lo, min(m, lo + chunk)))
        ref.moe_forward(olay, lay.x(m, offset=(b % nx) * m), rows=sel)
        rows += len(sel)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds or calls >= 10_000:
            return rows / el, rows, calls, el


def cpu_baseline(lay, m, seconds):
    v, rows, calls, el = oracle_rows_per_second(lay, m, seconds)
    return {"value": v, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{rows} rows of {m}-row batches in {calls} oracle calls "
                      f"(up to 8 rows evaluated per call, each call routing its whole batch), "
                      f"{el:.1f} s, numpy float64"}


def run_reference(args, cfg, m):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mixture_experts_decode_gemv_b200.synthetic import SyntheticLayer
    lay = SyntheticLayer(cfg)
    steps = args.steps if args.steps is not None else 20
    budget = 60.0   # seconds for the whole timed sample
    oracle_rows_per_second(lay, m, min(5.0, budget / 8))          # warm-up (decodes, BLAS)
    v, rows, calls, el = oracle_rows_per_second(lay, m, budget)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws,
        "steps": steps, "warmup": args.warmup, "ms_per_step": 1000.0 * m / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(cfg, m, ws),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)),
                         "kind": "oracle",
                         "sample": f"{rows} rows of {m}-row batches in {calls} oracle calls, "
                                   f"{el:.1f} s; a step is m rows, timed as m rows' share"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class Workload:
    """One layer on the device with its replicas, activation batches, workspace and output."""

    def __init__(self, cfg, m, dev0, lay, stream, replicas=None, reps=None):
        import torch
        from mixture_experts_decode_gemv_b200.synthetic import POOL_ROWS
        self.cfg, self.m, self.lay, self.stream = cfg, m, lay, stream
        self.dev0 = dev0
        self.nx = max(1, POOL_ROWS // m)
        self.xs = [dev0.x_to_device(lay.x(m, offset=i * m)) for i in range(self.nx)]
        self.ws = dev0.new_workspace(m, stream)
        self.out = dev0.new_out(m)
        active = []
        with torch.cuda.stream(stream):
            for i in range(self.nx):
                dev0.forward(self.xs[i], self.out, self.ws, stream=stream)
                active.append(dev0.read_routing(m, self.ws, stream)["active_count"])
        self.active = active
        self.bytes_per_batch = [touched_bytes(cfg, a) for a in active]
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        self.l2 = l2
        r_need = int(math.ceil(4 * l2 / max(1.0, min(self.bytes_per_batch)))) + 1
        if reps is not None and len(reps) >= r_need:
            self.reps = reps[:max(2, r_need)]
        else:
            layer_bytes = dev0.weight_bytes() + dev0.router_w.numel() * dev0.router_w.element_size()
            free, _ = torch.cuda.mem_get_info()
            r_cap = max(2, int(0.5 * free // max(1, layer_bytes)))
            R = max(2, min(r_need, r_cap)) if replicas is None else max(1, replicas)
            have = list(reps or [dev0])[:R]
            self.reps = have + [dev0.replica() for _ in range(R - len(have))]
        self.R = len(self.reps)

    def seq(self, n, start=0):
        return [((start + j) % self.R, (start + j) % self.nx) for j in range(n)]

    def call(self, r, i, x=None):
        self.reps[r].forward(self.xs[i] if x is None else x, self.out, self.ws, stream=self.stream)

    def capture(self, n):
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(self.stream):
            for r, i in self.seq(n):       # the exact launch sequence once outside capture
                self.call(r, i)
            with torch.cuda.graph(g, stream=self.stream):
                for r, i in self.seq(n):
                    self.call(r, i)
            g.replay()                     # a graph's first replay uploads it: keep it untimed
        return g

    def bytes_of(self, n):
        counts = np.bincount([i for _, i in self.seq(n)], minlength=self.nx)
        return float(np.dot(counts, self.bytes_per_batch))

    def time_windows(self, n, windows, wsz):
        """`windows` timed replays of one graph of n calls: milliseconds of each window."""
        import torch
        g = self.capture(n)
        torch.cuda.synchronize()
        ms = []
        for _ in range(windows):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier(wsz)
            torch.cuda.synchronize()
            with torch.cuda.stream(self.stream):
                a.record(self.stream)
                g.replay()
                b.record(self.stream)
            torch.cuda.synchronize()
            ms.append(max_over_ranks(a.elapsed_time(b), wsz))
        del g
        return ms


def summarise(wl, n, ms_list, peak):
    ms = statistics.median(ms_list)
    us = 1000.0 * ms / n
    gbs = wl.bytes_of(n) / (ms * 1e-3) / 1e9
    return {"us_per_layer": us, "tokens_per_s": wl.m * n / (ms * 1e-3),
            "touched_bytes_per_call": wl.bytes_of(n) / n, "hbm_gbs": gbs,
            "frac_of_measured_peak": gbs / peak, "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
            "window_us_per_layer": [1000.0 * t / n for t in ms_list]}


def run_ours(args, cfg, m):
    import torch
    from mixture_experts_decode_gemv_b200 import binding as B
    from mixture_experts_decode_gemv_b200.device_layer import DeviceLayer
    from mixture_experts_decode_gemv_b200.synthetic import CONFIGS, SyntheticLayer

    wsz, rank, local = dist_setup()
    B.moe_debug_set_path(1 if args.path == "chain" else 0)
    dev_index = torch.cuda.current_device()
    peak, peak_kind = measured_peaks()
    stream = torch.cuda.Stream()

    lay = SyntheticLayer(cfg)
    dev0 = DeviceLayer(lay, device=f"cuda:{dev_index}")
    wl = Workload(cfg, m, dev0, lay, stream, replicas=args.replicas)
    steps = args.steps if args.steps is not None else max(20, 2 * wl.R)
    steps = max(1, steps)

    # warm-up: W untimed steps
    with torch.cuda.stream(stream):
        for r, i in wl.seq(args.warmup):
            wl.call(r, i)
    torch.cuda.synchronize()

    clocks = ClockSampler(dev_index, enabled=not args.no_clocks)
    time.sleep(0.3)
    win_ms = wl.time_windows(steps, WINDOWS, wsz)     # each window: exactly `steps` calls
    clk = clocks.stop()
    ms = statistics.median(win_ms)
    status = dev0.device_status(wl.ws, stream)
    head = summarise(wl, steps, win_ms, peak)

    # end to end through the public call with host buffers (pinned), every step
    xh = [torch.empty_like(x, device="cpu").pin_memory() for x in wl.xs]
    for i in range(wl.nx):
        xh[i].copy_(wl.xs[i])
    xd = torch.empty_like(wl.xs[0])
    oh = torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(wsz)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for r, i in wl.seq(steps):
            xd.copy_(xh[i], non_blocking=True)
            wl.call(r, i, x=xd)
            oh.copy_(wl.out, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), wsz)

    # cold variant: L2 flushed (a write of twice its size) before every call, each timed alone
    cold_n = min(args.cold_steps, steps)
    cold_us = None
    if cold_n > 0:
        flush = torch.empty(2 * wl.l2, dtype=torch.uint8, device=f"cuda:{dev_index}")
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(cold_n)]
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for j, (a, b) in enumerate(evs):
                flush.fill_(j & 0xFF)
                a.record(stream)
                wl.call(j % wl.R, j % wl.nx)
                b.record(stream)
        torch.cuda.synchronize()
        cold_us = 1000.0 * statistics.median([a.elapsed_time(b) for a, b in evs])
        cold_us = 1000.0 * max_over_ranks(cold_us / 1000.0, wsz)
        del flush

    kernels_per_step = dev0.launches(m)
    result = {
        "metric": METRIC,
        "value": wsz * m * steps / (ms * 1e-3),
        "unit": "tokens/s",
        "n_gpus": wsz,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": ms / steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.x_dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": config_dict(cfg, m, wsz),
        "timing": {"windows": WINDOWS, "steps_per_window": steps, "replicas": wl.R,
                   "activation_batches": wl.nx, "l2_mib": wl.l2 >> 20,
                   "value_from": "median window"},
        **{k: v for k, v in head.items() if k != "tokens_per_s"},
        "roofline": {
            "bound": "hbm", "kernel": "whole layer call (its launches together)",
            "launches_per_step": kernels_per_step,
            "achieved": head["hbm_gbs"], "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": head["hbm_gbs"] / peak,
            "traffic": PROFILED_TRAFFIC.get((cfg.name, m)),
        },
        "e2e": {"value": wsz * m * steps / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": wl.xs[0].numel() * wl.xs[0].element_size(),
                "d2h_bytes_per_step": wl.out.numel() * wl.out.element_size(), "steps": steps},
        "gpu_launches": kernels_per_step * steps * WINDOWS,
        "clocks": clk,
        "cold": None if cold_us is None else {
            "us_per_layer_median": cold_us, "steps": cold_n,
            "policy": "L2 flushed by a write of 2x its size before every call; each call timed "
                      "alone with CUDA events; median"},
        "device_status": status,
    }
    head_reps = wl.reps
    del wl

    # the sweep: every published shape at each of its row counts, median of 5 windows each
    if not args.no_sweep:
        sweep = []
        clocks = ClockSampler(dev_index, enabled=not args.no_clocks)
        for name in SWEEP_CONFIGS:
            c = CONFIGS[name]
            if name == cfg.name:
                d0, ly, reps = dev0, lay, head_reps
            else:
                ly = SyntheticLayer(c)
                d0, reps = DeviceLayer(ly, device=f"cuda:{dev_index}"), None
            for mm in c.m_list:
                w = Workload(c, mm, d0, ly, stream, reps=reps)
                reps = w.reps
                n = w.R * max(1, int(math.ceil(args.sweep_steps / w.R)))
                with torch.cuda.stream(stream):
                    for r, i in w.seq(min(n, 3 * w.R)):
                        w.call(r, i)
                win = w.time_windows(n, WINDOWS, wsz)
                e = {"config": name, "m": mm, "weights": c.fmt, "launches": d0.launches(mm),
                     "active_experts_mean": float(np.mean(w.active)), "calls_per_window": n,
                     "replicas": w.R}
                e.update(summarise(w, n, win, peak))
                e["device_status"] = d0.device_status(w.ws, stream)
                sweep.append(e)
                del w
            if name == cfg.name:
                head_reps = None
            del d0, ly, reps
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        result["sweep"] = sweep
        result["sweep_clocks"] = clocks.stop()
    if rank == 0 and wsz == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(lay, m, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if wsz > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse_args()
    from mixture_experts_decode_gemv_b200.synthetic import CONFIGS
    cfg = CONFIGS[args.config]
    m = args.m if args.m is not None else (HEADLINE[1] if args.config == HEADLINE[0]
                                           else cfg.m_list[0])
    if m < 1 or m > 64:
        raise SystemExit("--m must be in 1..64")
    if args.impl == "reference":
        run_reference(args, cfg, m)
    else:
        run_ours(args, cfg, m)


if __name__ == "__main__":
    main()
