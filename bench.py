#!/usr/bin/env python
"""Benchmark: m=1 bf16 x NVFP4 decode GEMV on B200 (the serving-class decode shapes).

One step = the five serving decode shapes n x k in {2048x7168, 4096x4096, 4096x14336,
14336x4096, 10304x2688} at m=1 (PR #4038, "Split-K on the #3597 decode shapes", first
table), each called through the library's public op with the GEMV tactic at split-K
S in {1, 2, 4, 8, device-sized}: 25 calls. Every call is a CUDA-graph replay timed with
CUDA events on its stream, with L2 flushed (a 256 MiB read) before it, as decode serving
runs with a cold L2 (PR #4038, Performance: "Median GPU time over CUDA-graph replays with
a cold L2 cache"). The library's default tactic per shape is timed in a second pass and
reported beside the step.

value = algorithmic bytes of all calls / their summed device time (GB/s); algorithmic
bytes per call = n*k/2 + n*k/16 + 2*m*k + 2*m*n (packed codes, E4M3 scales, bf16 A and
out). Inputs are synthetic, seeded (A ~ N(0,1) in bf16, W ~ N(0, 0.02) quantised to NVFP4).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fi|reference]

N > 1 (torchrun, one rank per GPU): every rank runs the same workload on its own GPU
(replicas: the op has no exchange step); value = bytes of all ranks / max rank time.
--impl reference times the CPU oracle (the only reference implementation; there is no
upstream code to install) on the same workload and metric, on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/call and achieved HBM GB/s (% of B200 peak) for m=1 bf16×NVFP4 GEMV"
SHAPES = [(2048, 7168), (4096, 4096), (4096, 14336), (14336, 4096), (10304, 2688)]
SPLITS = [1, 2, 4, 8, 0]  # 0 = device-sized
M = 1
FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes per launch of the GEMV kernel (dram__bytes_read.sum + dram__bytes_write.sum)
# from one ncu capture per shape, keyed by the sha256 of the kernel source they were taken
# on; ignored (traffic = null) when the source has changed since.
NCU_TRAFFIC = {"source_sha256": None, "bytes": {}}


def algorithmic_bytes(m: int, n: int, k: int) -> int:
    return n * k // 2 + n * k // 16 + 2 * m * k + 2 * m * n


def _peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


def _gemv_source_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in ("gemv.cu", "common.cuh"):
        with open(os.path.join(ROOT, "bf16_activations_nvfp4_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# ------------------------------------------------------------------ clock sampling

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        self.file.flush()

    def summary(self) -> dict | None:
        try:
            with open(self.file.name) as f:
                rows = [[c.strip() for c in line.split(",")] for line in f if line.strip()]
            os.unlink(self.file.name)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------ fi arm

def run_fi(args, rank: int, world: int) -> dict | None:
    import torch
    import torch.distributed as dist

    import bf16_activations_nvfp4_b200 as fi
    from bf16_activations_nvfp4_b200 import inputs

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)

    def make_case(n, k, tactic, shared):
        info = fi.resolve_tactic(M, n, k, tactic)
        return dict(shared, n=n, k=k, tactic=tactic, info=info, bytes=algorithmic_bytes(M, n, k),
                    out=torch.empty((M, n), dtype=torch.bfloat16, device=dev))

    cases, defaults = [], []
    for n, k in SHAPES:
        W = torch.from_numpy(inputs.weights(n, k, seed=0)).to(dev)
        Wq, Ws, g = fi.pack_weights(W)
        del W
        a_host = inputs.activations(M, k, seed=0)
        shared = dict(Wq=Wq, Ws=Ws, g=g,
                      A=torch.from_numpy(a_host.view(np.int16)).view(torch.bfloat16).to(dev),
                      A_pinned=torch.from_numpy(a_host.view(np.int16)).view(torch.bfloat16).pin_memory(),
                      out_pinned=torch.empty((M, n), dtype=torch.bfloat16).pin_memory())
        for S in SPLITS:
            cases.append(make_case(n, k, fi.make_tactic(fi.KIND_GEMV, S, 0, 0), shared))
        defaults.append(make_case(n, k, fi.default_tactic(M, n, k), shared))
    ws_bytes = max(c["info"]["workspace_bytes"] for c in cases + defaults)
    ws = torch.empty(max(ws_bytes, 256) // 4 + 64, dtype=torch.float32, device=dev)
    fi.set_workspace(ws)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_out = torch.empty((), dtype=torch.int32, device=dev)
    torch.cuda.synchronize(dev)

    # one CUDA graph per shape holding the library call (1 or 2 kernels)
    with torch.cuda.stream(stream):
        for c in cases + defaults:
            fi.mm_bf16_fp4(c["A"], c["Wq"], c["Ws"], c["g"], tactic=c["tactic"], out=c["out"])
        torch.cuda.synchronize(dev)
        for c in cases + defaults:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                fi.mm_bf16_fp4(c["A"], c["Wq"], c["Ws"], c["g"], tactic=c["tactic"], out=c["out"])
            c["graph"] = graph
    torch.cuda.synchronize(dev)

    flush.fill_(1)

    def device_pass(steps: int, e2e: bool, cs=None):
        cs = cases if cs is None else cs
        evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in cs] for _ in range(steps)]
        with torch.cuda.stream(stream):
            for st in range(steps):
                for ci, c in enumerate(cs):
                    # evict L2 (2x its 126 MB) with a read, outside the timed interval; a read
                    # leaves clean lines, so no write-back lands inside the timed call
                    torch.amax(flush, dim=0, out=flush_out)
                    e0, e1 = evs[st][ci]
                    e0.record(stream)
                    if e2e:
                        c["A"].copy_(c["A_pinned"], non_blocking=True)
                        fi.mm_bf16_fp4(c["A"], c["Wq"], c["Ws"], c["g"], tactic=c["tactic"], out=c["out"])
                        c["out_pinned"].copy_(c["out"], non_blocking=True)
                    else:
                        c["graph"].replay()
                    e1.record(stream)
        return evs

    def times_us(evs):
        torch.cuda.synchronize(dev)
        return [[e0.elapsed_time(e1) * 1e3 for (e0, e1) in row] for row in evs]

    times_us(device_pass(args.warmup, False))
    times_us(device_pass(max(3, args.warmup // 2), True))

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        wall0 = time.perf_counter()
        dev_times = times_us(device_pass(args.steps, False))
        wall1 = time.perf_counter()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e2e_steps = max(5, args.steps // 4)
    e2e_times = times_us(device_pass(e2e_steps, True))
    def_times = times_us(device_pass(args.steps, False, defaults))

    total_us = sum(sum(row) for row in dev_times)
    e2e_total_us = sum(sum(row) for row in e2e_times)
    if world > 1:
        t = torch.tensor([total_us, e2e_total_us], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_us, e2e_total_us = float(t[0]), float(t[1])
    step_bytes = sum(c["bytes"] for c in cases)
    value = world * step_bytes * args.steps / (total_us * 1e-6) / 1e9
    e2e_value = world * step_bytes * e2e_steps / (e2e_total_us * 1e-6) / 1e9
    peaks = _peaks()
    launches_per_step = sum(1 + (c["info"]["splits"] > 1) for c in cases)

    if rank != 0:
        return None

    def summarize(cs, times):
        rows = []
        for ci, c in enumerate(cs):
            ts = [row[ci] for row in times]
            med = statistics.median(ts)
            gbs = c["bytes"] / (med * 1e-6) / 1e9
            info = c["info"]
            rows.append({"n": c["n"], "k": c["k"], "splits": info["splits"],
                         "requested_splits": fi.tactic_fields(c["tactic"])["splits"],
                         "rows_per_warp": info["variant"] & 0xF, "warps_per_row": info["variant"] >> 4,
                         "us_median": round(med, 3), "us_mean": round(statistics.fmean(ts), 3),
                         "gbs_median": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                         "tflops_median": round(2 * M * c["n"] * c["k"] / (med * 1e-6) / 1e12, 4)})
        return rows

    per_call = summarize(cases, dev_times)
    default_rows = summarize(defaults, def_times)
    def_total = sum(sum(row) for row in def_times)
    def_bytes = sum(c["bytes"] for c in defaults)
    achieved = step_bytes / (total_us / args.steps * 1e-6) / 1e9
    traffic = None
    if NCU_TRAFFIC["source_sha256"] == _gemv_source_sha() and NCU_TRAFFIC["bytes"]:
        traffic = statistics.fmean(NCU_TRAFFIC["bytes"].values())
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_us / args.steps / 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 x e2m1 (f16 products, f32 accumulate)",
        "data": "synthetic",
        "config": {
            "workload": "serving-class decode GEMV, m=1, n x k in " + ", ".join(f"{n}x{k}" for n, k in SHAPES),
            "m": M, "tactic": "GEMV, split-K S in {1,2,4,8,device-sized} per shape (25 calls per step)",
            "weights": "N(0,0.02) -> NVFP4",
            "activations": "N(0,1) -> bf16", "seed": 0,
            "l2": "flushed before every call (256 MiB read, outside the timed interval)",
            "timing": "CUDA-graph replay per call, CUDA events on the launching stream",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "us_per_call": {f"{p['n']}x{p['k']}": p["us_median"] for p in default_rows},
        "default_tactic": {"value": round(def_bytes * args.steps / (def_total * 1e-6) / 1e9, 2), "unit": "GB/s",
                           "per_shape": default_rows},
        "per_call": per_call,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": sum(2 * M * c["k"] for c in cases),
                "d2h_bytes_per_step": sum(2 * M * c["n"] for c in cases),
                "how": "public op on device weights; per call: pinned H2D copy of A, the op, D2H copy of out, "
                       "all between the CUDA events; L2 flushed before each call"},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "peak_source": peaks["source"] + " (copy bandwidth, burst)",
                     "note": "per library call: GEMV kernel plus the split-K reduce where the tactic splits"},
        "clocks": clocks.summary(),
        "wall_s_timed_region": round(wall1 - wall0, 3),
    }
    return line


# -------------------------------------------------------------- oracle (CPU) timing

def oracle_sample(target_s: float) -> dict:
    """Time the CPU oracle's product (dequantise + fp64 dot) on the same five shapes."""
    import oracle
    from bf16_activations_nvfp4_b200 import inputs

    packed = []
    for n, k in SHAPES:
        Wq, Ws, g = oracle.pack(inputs.weights(n, k, seed=0))
        packed.append((inputs.activations(M, k, seed=0), Wq, Ws, g, algorithmic_bytes(M, n, k)))
    reps, elapsed, nbytes = 0, 0.0, 0
    while elapsed < target_s and reps < 200:
        for A, Wq, Ws, g, b in packed:
            t0 = time.perf_counter()
            oracle.mm(A, Wq, Ws, g)
            elapsed += time.perf_counter() - t0
            nbytes += b
        reps += 1
    return {"value": round(nbytes / elapsed / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle", "reps": reps, "seconds": round(elapsed, 2),
            "sample": f"{reps} full passes over the five m=1 shapes (pack excluded)"}


def run_reference(args) -> dict:
    import oracle
    from bf16_activations_nvfp4_b200 import inputs

    packed = []
    for n, k in SHAPES:
        Wq, Ws, g = oracle.pack(inputs.weights(n, k, seed=0))
        packed.append((inputs.activations(M, k, seed=0), Wq, Ws, g, algorithmic_bytes(M, n, k)))
    # each step is one of the five products, in rotation, so K steps stay within minutes
    for st in range(args.warmup):
        A, Wq, Ws, g, _ = packed[st % len(packed)]
        oracle.mm(A, Wq, Ws, g)
    total, nbytes = 0.0, 0
    for st in range(args.steps):
        A, Wq, Ws, g, b = packed[st % len(packed)]
        t0 = time.perf_counter()
        oracle.mm(A, Wq, Ws, g)
        total += time.perf_counter() - t0
        nbytes += b
    value = nbytes / total / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "serving-class decode GEMV, m=1, n x k in " + ", ".join(f"{n}x{k}" for n, k in SHAPES),
                   "m": M, "seed": 0, "step": "one of the five products per step, in rotation"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{args.steps} steps, each one full m=1 product of one shape (rotating)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["fi", "reference"], default="fi")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=10.0)
    ap.add_argument("--shapes", default=None,
                    help="comma-separated n x k subset of the workload, e.g. 4096x14336 (profiling runs)")
    ap.add_argument("--splits", default=None, help="comma-separated subset of the split menu (0 = device-sized)")
    args = ap.parse_args(argv)
    global SHAPES, SPLITS
    if args.shapes:
        SHAPES = [tuple(int(v) for v in sh.split("x")) for sh in args.shapes.split(",")]
    if args.splits:
        SPLITS = [int(v) for v in args.splits.split(",")]
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = run_fi(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0 and line is not None:
        if world == 1 and args.cpu_baseline_seconds > 0:
            line["cpu_baseline"] = oracle_sample(args.cpu_baseline_seconds)
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
