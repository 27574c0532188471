#!/usr/bin/env python
"""Benchmark: m=1 bf16 x NVFP4 decode GEMV on B200 (the serving-class decode shapes).

Workload (PR #4038, "Split-K on the #3597 decode shapes", first table): the five serving
decode shapes n x k in {2048x7168, 4096x4096, 4096x14336, 14336x4096, 10304x2688} at m=1,
each called through the library's public op with the GEMV tactic at split-K
S in {1, 2, 4, 8, device-sized}. One step = those 25 calls.

Method (PR #4038, Description, "Performance": the pages time the median of CUDA-graph
replays with L2 cold, the way a serving stack runs):
  * the step is captured once as a CUDA graph; consecutive calls are chained with
    programmatic dependent launch, as in a decode step where one GEMV follows another;
  * L2 is kept cold without flushing by rotating every call over its own copy of the packed
    weights; the copies of each shape total >= 300 MB (> 2x the 126 MB L2), so no weight byte
    is in L2 when it is read (inputs larger than L2);
  * K replays of the step graph are timed with CUDA events on the launching stream;
  * per-call µs: a graph of repeated calls of one (shape, split) over its rotating copies.

value = algorithmic bytes of all calls / their device time (GB/s); algorithmic bytes per call
= n*k/2 + n*k/16 + 2*m*k + 2*m*n (packed codes, E4M3 scales, bf16 A and out). Synthetic
seeded inputs: A ~ N(0,1) in bf16, W ~ N(0, 0.02) quantised to NVFP4 by the library.

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
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/call and achieved HBM GB/s (% of B200 peak) for m=1 bf16×NVFP4 GEMV"
SHAPES = [(2048, 7168), (4096, 4096), (4096, 14336), (14336, 4096), (10304, 2688)]
SPLITS = [1, 2, 4, 8, 0]  # 0 = device-sized
M = 1
COLD_BYTES = 300 << 20  # per-shape footprint of the rotating weight copies
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes per launch of the GEMV kernel (dram__bytes_read.sum + dram__bytes_write.sum)
# from one ncu capture per shape, keyed by the sha256 of the kernel code they were taken on
# (comments excluded); ignored (traffic = null) when that code has changed since.
NCU_TRAFFIC = {"source_sha256": "a99dfc7674f8a00b7d7729ba7f7462fd7a114e51eaa244746630eceda2b810b4",
               "bytes": {"4096x14336": 33_109_760, "14336x4096": 33_083_648}}
# the roofline's dominant-kernel figure: the GEMV alone (split 1, one launch per call) on the
# two 33 MB serving shapes
ROOFLINE_SHAPES = [(4096, 14336), (14336, 4096)]


def algorithmic_bytes(m: int, n: int, k: int) -> int:
    return n * k // 2 + n * k // 16 + 2 * m * k + 2 * m * n


FALLBACK_BF16_TFLOPS = 1590.0
# lm_head-like GEMM (n=152064, k=5120): m=1 runs the GEMV, m=64 and m=256 the tensor-core path
LM_HEAD = (152064, 5120)
LM_HEAD_M = (1, 64, 256)


def _peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS, "source": "fallback"}


def run_lm_head(dev, stream, peaks) -> dict:
    """The lm_head-like workload at m in LM_HEAD_M, each timed as a CUDA graph of 5 calls (the
    438 MB of packed weights exceed L2, so every call streams them from HBM). The f16 tensor
    rate equals the bf16 one, so the tensor fraction is against the measured bf16 peak."""
    import torch

    import bf16_activations_nvfp4_b200 as fi
    from bf16_activations_nvfp4_b200 import inputs
    n, k = LM_HEAD
    W = torch.from_numpy(inputs.weights(n, k, seed=0, jitter=True)).to(dev)
    Wq, Ws, g = fi.pack_weights(W)
    del W
    ws_bytes = max(fi.workspace_bytes(m, n, k) for m in LM_HEAD_M)
    ws = torch.empty(max(ws_bytes, 256) // 4 + 64, dtype=torch.float32, device=dev)
    fi.set_workspace(ws)
    torch.cuda.synchronize(dev)
    rows = []
    for m in LM_HEAD_M:
        A = torch.from_numpy(inputs.activations(m, k, seed=0).view(np.int16)).view(torch.bfloat16).to(dev)
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        with torch.cuda.stream(stream):
            fi.mm_bf16_fp4(A, Wq, Ws, g, out=out)
            torch.cuda.synchronize(dev)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for _ in range(5):
                    fi.mm_bf16_fp4(A, Wq, Ws, g, out=out)
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize(dev)
            times = []
            for _ in range(5):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                times.append(e0.elapsed_time(e1) * 1e3 / 5)
        us = statistics.median(times)
        info = fi.resolve_tactic(m, n, k)
        flops, nbytes = 2 * m * n * k, algorithmic_bytes(m, n, k)
        rows.append({"m": m, "kind": "gemv" if info["kind"] == fi.KIND_GEMV else "mma", "us": round(us, 2),
                     "tflops": round(flops / us / 1e6, 1), "gbs": round(nbytes / us / 1e3, 1),
                     "frac_tensor": round(flops / us / 1e6 / peaks["bf16_tflops"], 4),
                     "frac_hbm": round(nbytes / us / 1e3 / peaks["hbm_gbs"], 4)})
        del graph, A, out
    return {"workload": f"lm_head-like GEMM n={n} k={k}, weights N(0,0.02) with per-row U(0.5,2) jitter",
            "peak_tflops": peaks["bf16_tflops"], "peak_source": peaks["source"] + " bf16 dense (cuBLAS, burst)",
            "per_m": rows}


def _strip_comments(src: str) -> str:
    """C/C++ source with its comments removed and each line's trailing blanks and the blank
    lines dropped, so that an edit to comments alone keeps the hash; string and character
    literals are kept as written."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


def _gemv_source_sha() -> str:
    """sha256 of the GEMV kernel's code (comments excluded) in gemv.cu and common.cuh."""
    import hashlib
    h = hashlib.sha256()
    for name in ("gemv.cu", "common.cuh"):
        with open(os.path.join(ROOT, "bf16_activations_nvfp4_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()


# ------------------------------------------------------------------ clock sampling

class ClockSampler:
    """NVML sampling (every 10 ms) of SM clock and throttle reasons while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None

    def _run(self, handle, nvml):
        while not self._stop.is_set():
            try:
                mhz = nvml.nvmlDeviceGetClockInfo(handle, nvml.NVML_CLOCK_SM)
                reasons = nvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            handle = nvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = nvml.nvmlDeviceGetMaxClockInfo(handle, nvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, args=(handle, nvml), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self) -> dict | None:
        if not self.samples:
            return None
        reasons = sorted({name for _, r in self.samples for name, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "NVML, 10 ms"}


# ------------------------------------------------------------------------ fi arm

def max_over_ranks(times_us: list[float], world: int, device=None) -> list[float]:
    """Element-wise maximum over ranks of per-rank device times (every rank calls this at
    the same point; a no-op on one rank)."""
    if world == 1:
        return list(times_us)
    import torch
    import torch.distributed as dist
    t = torch.tensor(times_us, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def replica_value(step_bytes: float, steps: int, world: int, time_us: float) -> float:
    """Whole-job GB/s of `world` replicas that each moved step_bytes per step for `steps`
    steps, over the slowest rank's device time."""
    return world * step_bytes * steps / (time_us * 1e-6) / 1e9


def run_fi(args, rank: int, world: int) -> dict | None:
    import torch
    import torch.distributed as dist

    import bf16_activations_nvfp4_b200 as fi
    from bf16_activations_nvfp4_b200 import inputs

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    peaks = _peaks()

    # ---- inputs: packed weights (with rotating copies), activations, outputs
    shapes = []
    for n, k in SHAPES:
        W = torch.from_numpy(inputs.weights(n, k, seed=0)).to(dev)
        Wq, Ws, g = fi.pack_weights(W)
        del W
        b = algorithmic_bytes(M, n, k)
        ncopy = max(len(SPLITS), -(-COLD_BYTES // b))
        copies = [(Wq, Ws)] + [(Wq.clone(), Ws.clone()) for _ in range(ncopy - 1)]
        a_host = inputs.activations(M, k, seed=0)
        shapes.append(dict(n=n, k=k, g=g, copies=copies, bytes=b,
                           A=torch.from_numpy(a_host.view(np.int16)).view(torch.bfloat16).to(dev),
                           A_pinned=torch.from_numpy(a_host.view(np.int16)).view(torch.bfloat16).pin_memory(),
                           out=torch.empty((M, n), dtype=torch.bfloat16, device=dev),
                           out_pinned=torch.empty((M, n), dtype=torch.bfloat16).pin_memory()))
    calls = []  # the step: every shape at every split
    for si, sh in enumerate(shapes):
        for ci, S in enumerate(SPLITS):
            t = fi.make_tactic(fi.KIND_GEMV, S, 0, 0)
            calls.append(dict(shape=si, copy=ci, tactic=t, info=fi.resolve_tactic(M, sh["n"], sh["k"], t)))
    defaults = [dict(shape=si, tactic=fi.default_tactic(M, sh["n"], sh["k"])) for si, sh in enumerate(shapes)]
    for d in defaults:
        sh = shapes[d["shape"]]
        d["info"] = fi.resolve_tactic(M, sh["n"], sh["k"], d["tactic"])
    ws_bytes = max(c["info"]["workspace_bytes"] for c in calls + defaults)
    ws = torch.empty(max(ws_bytes, 256) // 4 + 64, dtype=torch.float32, device=dev)
    fi.set_workspace(ws)
    torch.cuda.synchronize(dev)

    def call(si, copy, tactic):
        sh = shapes[si]
        Wq, Ws = sh["copies"][copy % len(sh["copies"])]
        fi.mm_bf16_fp4(sh["A"], Wq, Ws, sh["g"], tactic=tactic, out=sh["out"])

    def capture(fn):
        with torch.cuda.stream(stream):
            fn()  # warm-up outside capture (sets kernel attributes, checks arguments)
            torch.cuda.synchronize(dev)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                fn()
        torch.cuda.synchronize(dev)
        return graph

    def time_replays(graph, reps: int) -> list[float]:
        """Per-replay device time in us, each replay bracketed by events on the stream."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        with torch.cuda.stream(stream):
            for e0, e1 in evs:
                e0.record(stream)
                graph.replay()
                e1.record(stream)
        torch.cuda.synchronize(dev)
        return [e0.elapsed_time(e1) * 1e3 for e0, e1 in evs]

    # ---- the step graph (25 calls)
    step_graph = capture(lambda: [call(c["shape"], c["copy"], c["tactic"]) for c in calls])

    # ---- per-call graphs: one (shape, tactic) repeated over its rotating copies
    def per_call_graph(si, tactic):
        nrep = 2 * len(shapes[si]["copies"])
        return capture(lambda: [call(si, r, tactic) for r in range(nrep)]), nrep

    case_graphs = [per_call_graph(c["shape"], c["tactic"]) for c in calls]
    default_graphs = [per_call_graph(d["shape"], d["tactic"]) for d in defaults]

    time_replays(step_graph, args.warmup)
    for g_, _ in case_graphs + default_graphs:
        time_replays(g_, 2)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        wall0 = time.perf_counter()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                step_graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        wall1 = time.perf_counter()
        total_us = e0.elapsed_time(e1) * 1e3
        case_us = [statistics.median(time_replays(g_, 15)) / nrep for g_, nrep in case_graphs]
        default_us = [statistics.median(time_replays(g_, 15)) / nrep for g_, nrep in default_graphs]
    if world > 1:
        dist.barrier()
    lm_head = run_lm_head(dev, stream, peaks) if world == 1 and not args.no_lm_head else None
    extra = run_extra_shapes(dev, stream, peaks) if world == 1 and not args.no_lm_head else None

    # ---- end to end through the public op with host buffers (eager calls)
    e2e_steps = max(5, args.steps // 10)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for it in range(2 + e2e_steps):
            if it == 2:
                x0.record(stream)
            for c in calls:
                sh = shapes[c["shape"]]
                sh["A"].copy_(sh["A_pinned"], non_blocking=True)
                call(c["shape"], c["copy"], c["tactic"])
                sh["out_pinned"].copy_(sh["out"], non_blocking=True)
        x1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_us = x0.elapsed_time(x1) * 1e3

    # host cost per call on the 4096 x 14336 default: the public op (binding + C ABI) and the bare
    # C-ABI call with its arguments prepared once, each issued back to back without synchronising
    # (the launch queue absorbs them); the GPU work is the same in both
    host_us = {}
    with torch.cuda.stream(stream):
        hi = next((i for i, sh in enumerate(shapes) if (sh["n"], sh["k"]) == (4096, 14336)), 0)
        sh = shapes[hi]
        Wq, Ws = sh["copies"][0]
        t_def = fi.default_tactic(M, sh["n"], sh["k"])
        reps = 200
        for label in ("public_op", "c_abi"):
            torch.cuda.synchronize(dev)
            if label == "public_op":
                t0 = time.perf_counter()
                for _ in range(reps):
                    fi.mm_bf16_fp4(sh["A"], Wq, Ws, sh["g"], tactic=t_def, out=sh["out"])
                t1 = time.perf_counter()
            else:
                lib = fi.library()
                cargs = (sh["A"].data_ptr(), Wq.data_ptr(), Ws.data_ptr(), sh["g"].data_ptr(), sh["out"].data_ptr(),
                         M, sh["n"], sh["k"], t_def, stream.cuda_stream)
                t0 = time.perf_counter()
                for _ in range(reps):
                    lib.fi_mm_bf16_fp4(*cargs)
                t1 = time.perf_counter()
            host_us[label] = round((t1 - t0) / reps * 1e6, 2)
        torch.cuda.synchronize(dev)
    total_us, e2e_us = max_over_ranks([total_us, e2e_us], world, dev)
    step_bytes = sum(shapes[c["shape"]]["bytes"] for c in calls)
    value = replica_value(step_bytes, args.steps, world, total_us)
    e2e_value = replica_value(step_bytes, e2e_steps, world, e2e_us)
    launches_per_step = sum(1 + (c["info"]["splits"] > 1) for c in calls)
    if rank != 0:
        return None

    def row(si, info, tactic, us):
        sh = shapes[si]
        gbs = sh["bytes"] / (us * 1e-6) / 1e9
        return {"n": sh["n"], "k": sh["k"], "requested_splits": fi.tactic_fields(tactic)["splits"],
                "splits": info["splits"], "rows_per_stage": info["variant"] & 0xF,
                "us": round(us, 3), "gbs": round(gbs, 1),
                "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                "tflops": round(2 * M * sh["n"] * sh["k"] / (us * 1e-6) / 1e12, 4)}

    per_call = [row(c["shape"], c["info"], c["tactic"], us) for c, us in zip(calls, case_us)]
    default_rows = [row(d["shape"], d["info"], d["tactic"], us) for d, us in zip(defaults, default_us)]
    # dominant kernel: the GEMV alone (split 1: one launch per call, no reduce) on the 33 MB
    # shapes when they are in the workload, else on every shape
    key = lambda si: f"{shapes[si]['n']}x{shapes[si]['k']}"
    on = [c for c in calls if c["info"]["splits"] == 1]
    if any((shapes[c["shape"]]["n"], shapes[c["shape"]]["k"]) in ROOFLINE_SHAPES for c in on):
        on = [c for c in on if (shapes[c["shape"]]["n"], shapes[c["shape"]]["k"]) in ROOFLINE_SHAPES]
    s1 = [(shapes[c["shape"]]["bytes"], case_us[calls.index(c)]) for c in on]
    achieved = sum(b for b, _ in s1) / (sum(u for _, u in s1) * 1e-6) / 1e9
    traffic = None
    keys = [key(c["shape"]) for c in on]
    if NCU_TRAFFIC["source_sha256"] == _gemv_source_sha() and all(k_ in NCU_TRAFFIC["bytes"] for k_ in keys):
        traffic = round(statistics.fmean(NCU_TRAFFIC["bytes"][k_] for k_ in keys))
    kernels = {1: "gemv_stream_kernel", 2: "gemv_nvfp4_kernel", 3: "gemv_stream_kernel", 4: "gemv_reg_kernel",
               5: "gemv_lean_kernel"}
    roof_names = sorted({kernels.get(c["info"]["variant"] >> 4, "gemv") for c in on})
    roof_kernel = "/".join(roof_names) + ", split 1, one launch per call, on " + ", ".join(sorted(set(keys)))
    def_bytes = sum(shapes[d["shape"]]["bytes"] for d in defaults)
    return {
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
        "dtype": "bf16 x e2m1 (exact products, f32 accumulate)",
        "data": "synthetic",
        "config": {
            "workload": "serving-class decode GEMV, m=1, n x k in " + ", ".join(f"{n}x{k}" for n, k in SHAPES),
            "m": M, "calls_per_step": len(calls),
            "tactics": "GEMV at split-K S in {1,2,4,8,device-sized} for every shape",
            "weights": "N(0,0.02) -> NVFP4 (library pack)", "activations": "N(0,1) -> bf16", "seed": 0,
            "l2": "inputs larger than L2: the 25 calls of a step read 25 distinct weight copies (about 500 MB); per-call graphs rotate over >= 300 MB of copies per shape",
            "timing": "CUDA-graph replays (calls chained with programmatic dependent launch), CUDA events",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "us_per_call": {f"{r['n']}x{r['k']}": r["us"] for r in default_rows},
        "default_tactic": {"value": round(def_bytes / (sum(default_us) * 1e-6) / 1e9, 2), "unit": "GB/s",
                           "per_shape": default_rows},
        "per_call": per_call,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": sum(2 * M * shapes[c["shape"]]["k"] for c in calls),
                "d2h_bytes_per_step": sum(2 * M * shapes[c["shape"]]["n"] for c in calls),
                "how": "eager public-op calls; per call a pinned H2D copy of A, the op, a D2H copy of out",
                "host_us_per_call": dict(host_us, shape="4096x14336 default tactic",
                                         how="200 calls issued back to back, host wall time per call")},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "peak_source": peaks["source"] + " copy bandwidth (burst)",
                     "algorithmic_bytes_per_launch": round(statistics.fmean(b for b, _ in s1)),
                     "kernel": roof_kernel},
        "clocks": clocks.summary(),
        "wall_s_timed_region": round(wall1 - wall0, 3),
        "lm_head": lm_head,
        "decode_grid": extra,
    }


def run_extra_shapes(dev, stream, peaks) -> dict:
    """Default-tactic µs per call, cold L2 (each call reads its own weight copy, copies >= 300
    MB per shape), PDL-chained graph replays: the narrow-n decode grid at m = 1, the
    small-batch sweep of 4096 x 14336 at m in {1, 2, 4, 8, 16, 32}, and the second workload,
    the Qwen3.6-27B-shaped decode GEMMs at m = 1 (34816 x 5120, 5120 x 17408, 248320 x 5120)."""
    import torch

    import bf16_activations_nvfp4_b200 as fi
    from bf16_activations_nvfp4_b200 import inputs

    def time_case(m, n, k):
        W = torch.from_numpy(inputs.weights(n, k, seed=0)).to(dev)
        Wq, Ws, g = fi.pack_weights(W)
        del W
        b = algorithmic_bytes(m, n, k)
        wbytes = n * (k // 2 + k // 16)
        copies = [(Wq, Ws)] + [(Wq.clone(), Ws.clone()) for _ in range(-(-COLD_BYTES // wbytes) - 1)]
        A = torch.from_numpy(inputs.activations(m, k, seed=0, outliers=True).view(np.int16)).view(torch.bfloat16).to(dev)
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        t = fi.default_tactic(m, n, k)
        ws = torch.empty(max(fi.workspace_bytes(m, n, k, t), 256) // 4 + 64, dtype=torch.float32, device=dev)
        nrep = 2 * len(copies)
        with torch.cuda.stream(stream):
            fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=t, out=out, workspace=ws)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for r in range(nrep):
                    q, s_ = copies[r % len(copies)]
                    fi.mm_bf16_fp4(A, q, s_, g, tactic=t, out=out, workspace=ws)
            ts = []
            for _ in range(8):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3 / nrep)
        us = statistics.median(ts[2:])
        info = fi.resolve_tactic(m, n, k, t)
        del graph, copies
        return {"m": m, "n": n, "k": k, "us": round(us, 3), "gbs": round(b / (us * 1e-6) / 1e9, 1),
                "frac_hbm": round(b / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                "tflops": round(2 * m * n * k / us / 1e6, 3), "splits": info["splits"],
                "pipeline": info["variant"] >> 4 if info["kind"] == fi.KIND_GEMV else "mma"}

    narrow = [time_case(1, n, k) for n, k in inputs.NARROW_N]
    small = [time_case(m, *inputs.SMALL_BATCH_NK) for m in inputs.SMALL_BATCH_M]
    qwen = [time_case(1, n, k) for n, k in inputs.QWEN36_27B_DECODE]
    return {"narrow_n": narrow, "small_batch": small, "qwen36_27b_m1": qwen,
            "method": "default tactic, PDL-chained CUDA-graph replays over >= 300 MB of weight copies (cold L2)"}


def mma_wave(args) -> None:
    """Profiling cases for the tensor-core path, each timed over 10 eager calls after 3 warm-up
    calls with the default tactic, small enough for a multi-pass ncu capture of single
    launches: first the small-batch decode GEMM 4096 x 14336 at m = 8 (mma_nvfp4 launches 1-13),
    then one wave of CTAs (n = 148 x 256 rows, k = 5120, the lm_head-like k) at m = 64
    (launches 14-26) and m = 256 (launches 27-39)."""
    import torch

    import bf16_activations_nvfp4_b200 as fi
    from bf16_activations_nvfp4_b200 import inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n, k = inputs.SMALL_BATCH_NK
    W = torch.from_numpy(inputs.weights(n, k, seed=0)).to(dev)
    Wq, Ws, g = fi.pack_weights(W)
    del W
    m = 8
    fi.set_workspace(torch.empty(fi.workspace_bytes(m, n, k) // 4 + 64, dtype=torch.float32, device=dev))
    A = torch.from_numpy(inputs.activations(m, k, seed=0).view(np.int16)).view(torch.bfloat16).to(dev)
    out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        fi.mm_bf16_fp4(A, Wq, Ws, g, out=out)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(10):
        fi.mm_bf16_fp4(A, Wq, Ws, g, out=out)
    e1.record()
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / 10
    info = fi.resolve_tactic(m, n, k)
    print(json.dumps({"n": n, "k": k, "m": m, "kind": info["kind"], "splits": info["splits"],
                      "variant": info["variant"], "us": round(us, 2)}), flush=True)
    del Wq, Ws, A, out
    n, k = 148 * 256, LM_HEAD[1]
    W = torch.from_numpy(inputs.weights(n, k, seed=0)).to(dev)
    Wq, Ws, g = fi.pack_weights(W)
    del W
    ws = torch.empty(max(fi.workspace_bytes(m, n, k) for m in (64, 256)) // 4 + 64, dtype=torch.float32, device=dev)
    fi.set_workspace(ws)
    for m in (64, 256):
        A = torch.from_numpy(inputs.activations(m, k, seed=0).view(np.int16)).view(torch.bfloat16).to(dev)
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            fi.mm_bf16_fp4(A, Wq, Ws, g, out=out)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            fi.mm_bf16_fp4(A, Wq, Ws, g, out=out)
        e1.record()
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) * 1e3 / 10
        print(json.dumps({"n": n, "k": k, "m": m, "kind": fi.resolve_tactic(m, n, k)["kind"], "us": round(us, 2),
                          "tflops": round(2 * m * n * k / us / 1e6, 1)}), flush=True)


def sweep(args) -> None:
    """Print per-call µs of every listed tactic for each shape (cold-L2 graph method)."""
    import torch

    import bf16_activations_nvfp4_b200 as fi
    from bf16_activations_nvfp4_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    for n, k in SHAPES:
        W = torch.from_numpy(inputs.weights(n, k, seed=0)).to(dev)
        Wq, Ws, g = fi.pack_weights(W)
        del W
        b = algorithmic_bytes(args.m, n, k)
        copies = [(Wq, Ws)] + [(Wq.clone(), Ws.clone()) for _ in range(-(-COLD_BYTES // b) - 1)]
        A = torch.from_numpy(inputs.activations(args.m, k, seed=0).view(np.int16)).view(torch.bfloat16).to(dev)
        out = torch.empty((args.m, n), dtype=torch.bfloat16, device=dev)
        tactics = fi.list_tactics(args.m, n, k) + [fi.default_tactic(args.m, n, k)]
        ws = torch.empty(max(fi.workspace_bytes(args.m, n, k, t) for t in tactics) // 4 + 64, device=dev)
        for t in tactics:
            info = fi.resolve_tactic(args.m, n, k, t)
            nrep = 2 * len(copies)
            with torch.cuda.stream(stream):
                fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=t, out=out, workspace=ws)
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=stream):
                    for r in range(nrep):
                        q, s_ = copies[r % len(copies)]
                        fi.mm_bf16_fp4(A, q, s_, g, tactic=t, out=out, workspace=ws)
                ts = []
                for _ in range(12):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    graph.replay()
                    e1.record(stream)
                    e1.synchronize()
                    ts.append(e0.elapsed_time(e1) * 1e3 / nrep)
            us = statistics.median(ts[2:])
            print(json.dumps({"m": args.m, "n": n, "k": k, "tactic": fi.tactic_fields(t), "resolved": info,
                              "us": round(us, 3), "gbs": round(b / (us * 1e-6) / 1e9, 1)}), flush=True)
            del graph
        del copies


# -------------------------------------------------------------- oracle (CPU) timing

def _oracle_packed():
    import oracle
    from bf16_activations_nvfp4_b200 import inputs
    packed = []
    for n, k in SHAPES:
        Wq, Ws, g = oracle.pack(inputs.weights(n, k, seed=0))
        packed.append((inputs.activations(M, k, seed=0), Wq, Ws, g, algorithmic_bytes(M, n, k)))
    return packed


def _host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(target_s: float) -> dict:
    """The CPU oracle on the same five m = 1 shapes, once with 1 thread and once with every
    host core (os.sched_getaffinity), pack (fp32 quantiser) and matmul (fp64 dequantise + dot)
    timed separately per shape. `value` is the all-cores matmul rate in the metric's unit (GB/s
    of algorithmic bytes); passes repeat until about target_s seconds of matmul time per thread
    count, each shape's pack is timed once per thread count."""
    import oracle
    from bf16_activations_nvfp4_b200 import inputs
    cores = _host_cores()
    data = [(n, k, inputs.weights(n, k, seed=0), inputs.activations(M, k, seed=0), algorithmic_bytes(M, n, k))
            for n, k in SHAPES]
    per_shape = {f"{n}x{k}": {"n": n, "k": k} for n, k, *_ in data}
    rates = {}
    for label, threads in (("1_thread", 1), ("all_cores", cores)):
        oracle.set_num_threads(threads)
        packed = []
        for n, k, W, A, b in data:
            t0 = time.perf_counter()
            Wq, Ws, g = oracle.pack(W)
            per_shape[f"{n}x{k}"][f"pack_ms_{label}"] = round((time.perf_counter() - t0) * 1e3, 2)
            packed.append((n, k, A, Wq, Ws, g, b))
        reps, elapsed, nbytes = 0, 0.0, 0
        mm_s = {f"{n}x{k}": [] for n, k, *_ in data}
        while elapsed < target_s / 2 and reps < 200:
            for n, k, A, Wq, Ws, g, b in packed:
                t0 = time.perf_counter()
                oracle.mm(A, Wq, Ws, g)
                dt = time.perf_counter() - t0
                mm_s[f"{n}x{k}"].append(dt)
                elapsed += dt
                nbytes += b
            reps += 1
        for key, ts in mm_s.items():
            per_shape[key][f"matmul_ms_{label}"] = round(statistics.median(ts) * 1e3, 3)
        rates[label] = {"value": round(nbytes / elapsed / 1e9, 4), "unit": "GB/s", "threads": threads,
                        "reps": reps, "matmul_seconds": round(elapsed, 2)}
    oracle.set_num_threads(cores)
    return {"value": rates["all_cores"]["value"], "unit": "GB/s", "cores": cores, "kind": "oracle",
            "one_thread": rates["1_thread"], "all_cores": rates["all_cores"],
            "per_shape": list(per_shape.values()),
            "sample": f"{rates['all_cores']['reps']} full passes over the five m=1 products at {cores} threads "
                      f"({rates['1_thread']['reps']} at 1 thread); pack timed once per shape and thread count"}


REFERENCE_BUDGET_S = 120.0  # whole --impl reference run, all steps


def run_reference(args) -> dict:
    """The oracle on the same workload: each step is one shape's m=1 product, in rotation,
    over an evenly spaced sample of output columns sized so that all K + W steps take about
    REFERENCE_BUDGET_S; the bytes counted are the sampled columns' share of the call."""
    import numpy as np

    import oracle
    packed = _oracle_packed()
    per_step = REFERENCE_BUDGET_S / (args.steps + args.warmup)
    plans = []
    for A, Wq, Ws, g, b in packed:
        n = Wq.shape[0]
        t0 = time.perf_counter()
        oracle.mm(A, Wq, Ws, g, cols=np.arange(0, n, 16))  # a 1/16 probe of the full cost
        full_s = (time.perf_counter() - t0) * 16
        ncols = max(1, min(n, int(n * per_step / max(full_s, 1e-9))))
        cols = np.unique(np.linspace(0, n - 1, ncols).round().astype(np.int64))
        plans.append((A, Wq, Ws, g, cols, b * cols.size / n))
    for st in range(args.warmup):
        A, Wq, Ws, g, cols, _ = plans[st % len(plans)]
        oracle.mm(A, Wq, Ws, g, cols=cols)
    total, nbytes = 0.0, 0.0
    for st in range(args.steps):
        A, Wq, Ws, g, cols, b = plans[st % len(plans)]
        t0 = time.perf_counter()
        oracle.mm(A, Wq, Ws, g, cols=cols)
        total += time.perf_counter() - t0
        nbytes += b
    value = nbytes / total / 1e9
    frac = sum(p[4].size / p[1].shape[0] for p in plans) / len(plans)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "serving-class decode GEMV, m=1, n x k in " + ", ".join(f"{n}x{k}" for n, k in SHAPES),
                   "m": M, "seed": 0,
                   "step": "one of the five products per step, in rotation, over a column sample"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{args.steps} steps, each one shape's m=1 product (rotating) over an evenly "
                                   f"spaced {frac:.1%} of its output columns on average"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["fi", "reference"], default="fi")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=10.0)
    ap.add_argument("--shapes", default=None,
                    help="comma-separated n x k subset of the workload, e.g. 4096x14336 (profiling runs)")
    ap.add_argument("--splits", default=None, help="comma-separated subset of the split menu (0 = device-sized)")
    ap.add_argument("--sweep", action="store_true", help="print per-call µs of every listed tactic and exit")
    ap.add_argument("--m", type=int, default=1, help="activation rows for --sweep")
    ap.add_argument("--no-lm-head", action="store_true", help="skip the lm_head-like GEMM measurement")
    ap.add_argument("--mma-wave", action="store_true",
                    help="profiling case: the tensor-core path on one wave of CTAs at m = 64 and 256, then exit")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    global SHAPES, SPLITS
    if args.shapes:
        SHAPES = [tuple(int(v) for v in sh.split("x")) for sh in args.shapes.split(",")]
    if args.splits:
        SPLITS = [int(v) for v in args.splits.split(",")]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if args.sweep:
        sweep(args)
        return 0
    if args.mma_wave:
        mma_wave(args)
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
