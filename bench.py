#!/usr/bin/env python
"""Throughput of the packed 4-bit weight path on B200.

Headline workload: the FP4-G16 (fp16 group scale) GEMV at the Mamba-2 8B
in_proj shape, n = 18560, k = 4096, one decode token (m = 1).  A step is one
call of the fused dequantise-and-multiply (stream packed blocks, decode,
multiply-accumulate, reduce, store y) for one token.  ``value`` is packed
weight bytes per second over all ranks.  The other workloads of the path
(m = 4/16 sweeps, IQ4_NL, dequantisation, prefill GEMM, routed experts) are
measured the same way and reported under ``workloads``.

Timing: W untimed warm-up steps, then K steps replayed from a CUDA graph of
back-to-back launches, bracketed by a barrier and synchronisation, timed with
CUDA events on the launching stream, max over ranks.  The weights rotate over
enough device copies to exceed 4x the L2 size, so every step streams from HBM.

``--impl reference`` times the CPU oracle (plain C, one host thread) on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "packed 4-bit GEMV weight GB/s vs HBM peak (M=1); prefill GEMM TFLOP/s (M=2048)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# ncu DRAM traffic per launch (read + write bytes) of the dominant kernel, by
# variant string; a variant not listed here reports traffic null.
TRAFFIC = {}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clk", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [s.strip() for s in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        # samples under load: the top half of the clocks seen (the sampler
        # starts slightly before and ends slightly after the timed region)
        loaded = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; the path itself shards with no
# collective: every rank runs independent replicas of the workload)
# ---------------------------------------------------------------------------
def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    import torch
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------
def l2_bytes():
    import torch
    return int(torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size)


def rotating_copies(nbytes: int, l2: int, cap_bytes: int = 6 << 30) -> int:
    r = max(2, math.ceil(4 * l2 / max(nbytes, 1)))
    return max(1, min(r, cap_bytes // max(nbytes, 1)))


def graph_of(launch, count: int):
    """Capture `count` calls of launch(i) into one CUDA graph."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(min(count, 3)):  # warm outside capture (descriptor encode, attributes)
            launch(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(count):
            launch(i)
    torch.cuda.synchronize()
    return g


def time_graph(g, reps: int, world: int, sampler=None):
    """Replay `g` reps times; returns (seconds, clocks dict or None)."""
    import torch
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(reps):
        g.replay()
    e1.record(st)
    e1.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    barrier(world)
    return e0.elapsed_time(e1) / 1e3, clocks


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def gemv_workload(p, x_bits, steps, warmup, world, l2, sampler=None, graph_len=100):
    """Device-resident GEMV throughput; returns dict."""
    import torch
    from packed_bit_weight_b200 import qmm
    base = qmm.PackedWeights.from_host(p)
    R = rotating_copies(base.nbytes, l2)
    ws = [base] + [qmm.PackedWeights(base.fmt, base.n, base.k, base.data.clone(),
                                     None if base.scales is None else base.scales.clone(), base.global_scale)
                   for _ in range(R - 1)]
    m = x_bits.shape[0]
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    y = torch.empty((m, p.n), dtype=torch.int16, device="cuda")

    def launch(i):
        qmm.qmm_gemv(ws[i % R], x, y)

    glen = max(1, min(graph_len, steps))
    g = graph_of(launch, glen)
    variant = qmm.qmm_last_variant()
    wreps = max(1, math.ceil(warmup / glen))
    time_graph(g, wreps, world)
    reps = max(1, steps // glen)
    secs, clocks = time_graph(g, reps, world, sampler)
    launches = reps * glen
    assert qmm.qmm_sync_check() == 0
    per = secs / launches
    del g
    return {"variant": variant, "launches": launches, "seconds": secs, "s_per_launch": per,
            "bytes_per_launch": base.nbytes, "gbs": base.nbytes / per / 1e9, "copies": R,
            "rotating_bytes": R * base.nbytes, "clocks": clocks, "m": m, "n": p.n, "k": p.k}


def gemv_e2e(p, x_bits, steps, world):
    """Same GEMV through the public Python API with host buffers: pinned x
    host->device, the call, y device->host, every step."""
    import torch
    from packed_bit_weight_b200 import qmm
    w = qmm.PackedWeights.from_host(p)
    m = x_bits.shape[0]
    xh = torch.from_numpy(x_bits.view(np.int16).copy()).pin_memory()
    yh = torch.empty((m, p.n), dtype=torch.int16).pin_memory()
    xd = torch.empty_like(xh, device="cuda")
    yd = torch.empty((m, p.n), dtype=torch.int16, device="cuda")

    def step():
        xd.copy_(xh, non_blocking=True)
        qmm.qmm_gemv(w, xd, yd)
        yh.copy_(yd, non_blocking=True)

    for _ in range(20):
        step()
    torch.cuda.synchronize()
    barrier(world)
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        step()
    e1.record(st)
    e1.synchronize()
    secs = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    return {"seconds": secs, "steps": steps, "h2d": xh.numel() * 2, "d2h": yh.numel() * 2,
            "gbs": world * w.nbytes * steps / secs / 1e9}


def cpu_oracle_gemv(p, x_bits, budget_s=10.0, rows=None):
    """The oracle as it stands, one host thread, on a bounded row sample."""
    import oracle
    rows = rows or max(16, p.n // 4)
    rows = min(rows, p.n)
    sub = type(p)(p.fmt, rows, p.k, p.data[: oracle.data_bytes(p.fmt, rows, p.k)],
                  None if p.scales is None else p.scales[: oracle.scale_bytes(p.fmt, rows, p.k)], p.global_scale)
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.matmul(sub.fmt, sub.n, sub.k, sub.data, sub.scales, sub.global_scale, x_bits)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": sub.nbytes * reps / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d of %d rows x %d reps (%.1f s, one thread)" % (rows, p.n, reps, dt)}


def extra_workloads(args, world, l2, peaks):
    """Every other workload of the path, device-resident, kernel throughput."""
    from packed_bit_weight_b200 import synth
    out = {}
    steps = max(200, args.steps // 10)
    warm = max(3, args.warmup // 10)
    mats = synth.make_sweep()
    for name, (p, xall) in mats.items():
        for m in (1, 4, 16):
            r = gemv_workload(p, xall[:m], steps, warm, world, l2)
            out["fp4g16_gemv_%s_m%d" % (name, m)] = {
                "variant": r["variant"], "gbs": r["gbs"], "frac_hbm": r["gbs"] / peaks["hbm_gbs"],
                "us_per_launch": r["s_per_launch"] * 1e6, "tflops": 2 * m * p.n * p.k / r["s_per_launch"] / 1e12}
    p, x = synth.make_gemv(synth.FP4_IN_PROJ, synth.FMT_FP4G16_E4M3)
    r = gemv_workload(p, x, steps, warm, world, l2)
    out["fp4g16_e4m3_gemv_in_proj_m1"] = {"variant": r["variant"], "gbs": r["gbs"],
                                          "frac_hbm": r["gbs"] / peaks["hbm_gbs"],
                                          "us_per_launch": r["s_per_launch"] * 1e6}
    p, x = synth.make_gemv(synth.IQ4_TINY)
    r = gemv_workload(p, x, steps, warm, world, l2)
    out["iq4nl_gemv_tiny_256x512_m1"] = {"variant": r["variant"], "gbs": r["gbs"],
                                         "us_per_launch": r["s_per_launch"] * 1e6, "note": "fits in L2"}
    return out


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=500)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="headline workload only")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from packed_bit_weight_b200 import synth
    wl = synth.FP4_IN_PROJ
    config = {"workload": wl.name, "format": "FP4-G16 (E2M1 codes, fp16 scale per 16 k)", "n": 18560, "k": 4096,
              "m": 1, "seed": wl.seed, "parallelism": "replicas"}

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        p, x = synth.make_gemv(wl)
        cb = cpu_oracle_gemv(p, x, budget_s=args.cpu_budget)
        steps = args.steps
        line = {"metric": METRIC, "value": cb["value"], "unit": "GB/s", "n_gpus": world, "steps": steps,
                "warmup": args.warmup, "ms_per_step": p.nbytes / (cb["value"] * 1e9) * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config, "impl": "reference", "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                "gpu_launches": 0}
        print(json.dumps(line))
        return 0

    world, rank, local = dist_init()
    import torch
    from packed_bit_weight_b200 import qmm  # noqa: F401  (fails loudly if the library is missing)
    peaks, peak_src = load_peaks()
    l2 = l2_bytes()
    p, x = synth.make_gemv(wl)
    sampler = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                           if "CUDA_VISIBLE_DEVICES" in os.environ else local)
    r = gemv_workload(p, x, args.steps, args.warmup, world, l2, sampler)
    secs = max_over_ranks(r["seconds"], world)
    launches = r["launches"]
    value = world * r["bytes_per_launch"] * launches / secs / 1e9
    per_launch = secs / launches
    achieved = r["bytes_per_launch"] / per_launch / 1e9
    e2e = gemv_e2e(p, x, max(200, min(5000, args.steps // 4)), world)
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": launches,
            "warmup": args.warmup, "ms_per_step": per_launch * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp16-in/fp32-acc (4-bit packed weights)", "data": "synthetic",
            "config": dict(config, l2="rotating %d weight copies = %.0f MB > 4x L2 (%d MB)" %
                           (r["copies"], r["rotating_bytes"] / 1e6, l2 >> 20),
                           timing="CUDA graph of 100 back-to-back launches, replayed"),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": TRAFFIC.get(r["variant"]),
                         "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_src if peak_src == "measured"
                         else "fallback 6650 GB/s", "kernel": r["variant"],
                         "algorithmic_bytes_per_launch": r["bytes_per_launch"]},
            "clocks": r["clocks"],
            "e2e": {"value": round(e2e["gbs"], 2), "unit": "GB/s", "h2d_bytes_per_step": e2e["h2d"],
                    "d2h_bytes_per_step": e2e["d2h"]},
            "gpu_launches": launches}
    if not args.no_extra:
        line["workloads"] = extra_workloads(args, world, l2, peaks)
    if rank == 0:
        line["cpu_baseline"] = cpu_oracle_gemv(p, x, budget_s=args.cpu_budget) if world == 1 else None
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
