#!/usr/bin/env python
"""Throughput of the decode-time MoE layer on B200: µs/layer, tokens/s and HBM GB/s.

One step = one call of the whole layer (router GEMV, top-k routing, grouping by expert,
gate+up+SwiGLU, down projection with the weighted blend and shared expert) on m rows of a seeded
synthetic layer. Steps rotate over R replicas of the layer's weights (same values, separate
device memory) and over the 64-row activation pool, so the weights touched between two uses of
a replica exceed 4x the L2 cache: every timed call streams its weights from HBM.

Default workload: the Qwen3-30B-A3B-shaped layer (hidden 2048, 128 experts, top-8,
moe_intermediate 768, bf16 weights) at m = 1.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--m M]
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

# DRAM bytes per launch of the kernel that runs the call (dram__bytes_read.sum +
# dram__bytes_write.sum, one ncu capture of the current kernel; see profiles/). Keyed by
# (workload config name, m, launches per call); absent keys report null.
PROFILED_TRAFFIC = {
    ("qwen3_30b_a3b", 1, 1): 77.6e6,  # profiles/moe_fused_kernel_qwen3_30b_a3b_m1.md
}
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", default="qwen3_30b_a3b")
    ap.add_argument("--m", type=int, default=1)
    ap.add_argument("--graph-len", type=int, default=128)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cold-steps", type=int, default=50,
                    help="calls timed one by one after an L2 flush (0: skip)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--path", choices=("auto", "chain"), default="auto",
                    help="launch path: automatic (persistent kernel for m <= 4) or the chain")
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
        self.gpu = gpu_index
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
            + f", {cfg.fmt} weights, {cfg.routing} routing")


def cpu_baseline(lay, m, seconds, nx):
    """The float64 oracle, as it stands, on a bounded sample of the same workload."""
    from oracle import moe_ref as ref
    olay = ref.OracleLayer(lay)
    calls, t0 = 0, time.perf_counter()
    while True:
        x = lay.x(m, offset=(calls % nx) * m)
        ref.moe_forward(olay, x)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds or calls >= 10_000:
            break
    cores = len(os.sched_getaffinity(0))
    return {"value": m * calls / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{calls} oracle calls of {m} row(s) on activation batches 0..{min(calls, nx) - 1}"
                      f" of the same layer, {el:.1f} s, numpy float64"}


def run_reference(args, cfg):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mixture_experts_decode_gemv_b200.synthetic import POOL_ROWS, SyntheticLayer
    from oracle import moe_ref as ref
    m = args.m
    lay = SyntheticLayer(cfg)
    nx = max(1, POOL_ROWS // m)
    olay = ref.OracleLayer(lay)
    steps = args.steps if args.steps is not None else 20
    budget = 150.0  # seconds for warm-up + timed steps together
    per_step_budget = budget / max(1, steps + args.warmup)
    t_w = time.perf_counter()
    for i in range(min(args.warmup, 3)):
        ref.moe_forward(olay, lay.x(m, offset=(i % nx) * m))
        if time.perf_counter() - t_w > budget / 4:
            break
    calls, t0 = 0, time.perf_counter()
    while True:
        ref.moe_forward(olay, lay.x(m, offset=(calls % nx) * m))
        calls += 1
        el = time.perf_counter() - t0
        if el >= per_step_budget * steps or calls >= steps:
            break
    value = m * calls / el
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": steps, "warmup": args.warmup, "ms_per_step": 1000.0 * el / calls,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_name(cfg, m), "m": m},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{calls} oracle calls of {m} row(s) within a "
                                   f"{per_step_budget * steps:.0f} s budget"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, cfg):
    import torch
    from mixture_experts_decode_gemv_b200.device_layer import DeviceLayer
    from mixture_experts_decode_gemv_b200.synthetic import POOL_ROWS, SyntheticLayer

    wsz, rank, local = dist_setup()
    from mixture_experts_decode_gemv_b200 import binding as B
    B.moe_debug_set_path(1 if args.path == "chain" else 0)
    dev_index = torch.cuda.current_device()
    m = args.m
    lay = SyntheticLayer(cfg)
    dev0 = DeviceLayer(lay, device=f"cuda:{dev_index}")
    nx = max(1, POOL_ROWS // m)
    xs = [dev0.x_to_device(lay.x(m, offset=i * m)) for i in range(nx)]
    stream = torch.cuda.Stream()
    ws = dev0.new_workspace(m, stream)
    out = dev0.new_out(m)

    # distinct experts per activation batch, from the library's own routing
    active = []
    with torch.cuda.stream(stream):
        for i in range(nx):
            dev0.forward(xs[i], out, ws, stream=stream)
            active.append(dev0.read_routing(m, ws, stream)["active_count"])
    bytes_per_batch = [touched_bytes(cfg, a) for a in active]
    mean_bytes = float(np.mean(bytes_per_batch))

    l2 = torch.cuda.get_device_properties(dev_index).L2_cache_size
    layer_bytes = dev0.weight_bytes() + dev0.router_w.numel() * dev0.router_w.element_size()
    free, _ = torch.cuda.mem_get_info(dev_index)
    r_need = int(math.ceil(4 * l2 / max(1.0, min(bytes_per_batch)))) + 1
    r_cap = max(2, int(0.6 * free // max(1, layer_bytes)))
    R = max(2, min(r_need, r_cap)) if args.replicas is None else max(1, args.replicas)
    reps = [dev0] + [dev0.replica() for _ in range(R - 1)]

    G = R * max(1, int(math.ceil(args.graph_len / R)))
    est_us = mean_bytes / 6.0e6 + 5.0            # ~6 TB/s plus fixed latency, for sizing only
    steps = args.steps if args.steps is not None else max(G, int(2.0e6 / est_us))
    steps = max(1, steps)

    def seq(n, start=0):
        return [((start + j) % R, (start + j) % nx) for j in range(n)]

    def capture(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for r, i in seq(n):  # warm the exact launch sequence once outside capture
                reps[r].forward(xs[i], out, ws, stream=stream)
            with torch.cuda.graph(g, stream=stream):
                for r, i in seq(n):
                    reps[r].forward(xs[i], out, ws, stream=stream)
        return g

    n_full, rem = divmod(steps, G)
    g_full = capture(G) if n_full else None
    g_rem = capture(rem) if rem else None
    with torch.cuda.stream(stream):  # a graph's first replay uploads it: keep that untimed
        for g in (g_full, g_rem):
            if g is not None:
                g.replay()
    torch.cuda.synchronize()

    # warm-up: W untimed steps
    with torch.cuda.stream(stream):
        for r, i in seq(args.warmup):
            reps[r].forward(xs[i], out, ws, stream=stream)
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(wsz)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev_index, enabled=not args.no_clocks)
    time.sleep(0.3)
    with torch.cuda.stream(stream):  # graphs replay on the current stream: keep it `stream`
        start.record(stream)
        for _ in range(n_full):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
        end.record(stream)
    torch.cuda.synchronize()
    barrier(wsz)
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    ms = max_over_ranks(ms, wsz)
    status = dev0.device_status(ws, stream)

    # algorithmic bytes of the timed calls (batch i of call j is j % nx)
    counts = np.bincount([i for _, i in seq(steps)], minlength=nx)
    bytes_timed = float(np.dot(counts, bytes_per_batch))
    us_per_step = 1000.0 * ms / steps
    gbs = bytes_timed / (ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()

    # end to end through the public call with host buffers
    e2e_steps = min(args.e2e_steps, steps)
    xh = [torch.empty_like(x, device="cpu").pin_memory() for x in xs]
    for i in range(nx):
        xh[i].copy_(xs[i])
    xd = torch.empty_like(xs[0])
    oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(wsz)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for r, i in seq(e2e_steps):
            xd.copy_(xh[i], non_blocking=True)
            reps[r].forward(xd, out, ws, stream=stream)
            oh.copy_(out, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), wsz)

    # cold variant: L2 flushed (a write of twice its size) before every call, each call timed
    # on its own; the median is reported beside the rotating-replica figure
    cold_n = min(args.cold_steps, steps)
    cold_us = None
    if cold_n > 0:
        flush = torch.empty(2 * l2, dtype=torch.uint8, device=f"cuda:{dev_index}")
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(cold_n)]
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for j, (a, b) in enumerate(evs):
                flush.fill_(j & 0xFF)
                a.record(stream)
                reps[j % R].forward(xs[j % nx], out, ws, stream=stream)
                b.record(stream)
        torch.cuda.synchronize()
        cold_us = 1000.0 * statistics.median([a.elapsed_time(b) for a, b in evs])
        cold_us = 1000.0 * max_over_ranks(cold_us / 1000.0, wsz)
        del flush

    kernels_per_step = dev0.launches(m)
    kernel_name = ("moe_fused_kernel (whole layer, one persistent launch)" if kernels_per_step == 1
                   else "whole layer (router_topk_group + gate_up_swiglu + down_blend, PDL)")
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
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": workload_name(cfg, m), "m": m, "weights": cfg.fmt,
            "replicas": R, "layer_bytes": layer_bytes,
            "l2_policy": f"inputs larger than L2: {R} weight replicas x {nx} activation batches "
                         f"rotate, >= 4x L2 ({l2 >> 20} MiB) between reuses",
            "parallelism": f"replicas x{wsz}",
        },
        "us_per_layer": us_per_step,
        "touched_bytes_per_step": bytes_timed / steps,
        "hbm_gbs": gbs,
        "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
        "roofline": {
            "bound": "hbm", "kernel": kernel_name, "launches_per_step": kernels_per_step,
            "achieved": gbs, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": gbs / peak,
            "traffic": PROFILED_TRAFFIC.get((cfg.name, m, kernels_per_step)),
        },
        "e2e": {"value": wsz * m * e2e_steps / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": xs[0].numel() * xs[0].element_size(),
                "d2h_bytes_per_step": out.numel() * out.element_size(), "steps": e2e_steps},
        "gpu_launches": kernels_per_step * steps,
        "clocks": clk,
        "cold": None if cold_us is None else {
            "us_per_layer_median": cold_us, "steps": cold_n,
            "policy": "L2 flushed by a write of 2x its size before every call; each call timed "
                      "alone with CUDA events; median"},
        "device_status": status,
    }
    if rank == 0 and wsz == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(lay, m, args.cpu_seconds, nx)
    if rank == 0:
        print(json.dumps(result), flush=True)
    del g_full, g_rem
    if wsz > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse_args()
    from mixture_experts_decode_gemv_b200.synthetic import CONFIGS
    cfg = CONFIGS[args.config]
    if args.m < 1 or args.m > 64:
        raise SystemExit("--m must be in 1..64")
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
