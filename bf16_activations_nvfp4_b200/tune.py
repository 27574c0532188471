"""Offline cold-L2 tuner: measures every listed tactic per (shape, m bucket) on this GPU and
writes the default-tactic table the library compiles in (csrc/tactic_table.inc).

    python -m bf16_activations_nvfp4_b200.tune [--shapes 4096x14336,...] [--out PATH]

After PR #4038 (Description and Reviewer Notes): the op carries a per-shape tactic choice, and
a tuner that ranks tactics with the weights warm in L2 over-ranks split tactics, which mis-picked
cells on the pages' own GPUs. So every candidate here is timed the way a decode step runs it:
each call reads its own copy of the packed weights (copies rotate over more than twice the L2),
calls are chained by programmatic dependent launch inside one CUDA graph, and the median of the
graph replays is taken. The fastest tactic of a bucket over the bucket's sample m values wins; a
bucket's tactic is one code for all of its m, so the default stays batch-invariant inside it.

Buckets of m: {1}, {2}, {3..4}, {5..32}, {33..256} ({2} apart: on B200 the GEMV's register
pipeline wins at m = 2 where the tensor-core path wins at m = 4 on the 4096 x 14336 class of
shapes). Candidates are the codes fi_list_tactics offers at every sample m of the bucket. The table is keyed by (n, k, SM count); shapes and devices it
does not list fall back to the library's built-in rules.
"""
from __future__ import annotations

import argparse
import datetime
import os
import statistics
import sys

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
OUT = os.path.join(PKG, "csrc", "tactic_table.inc")

# (m_lo, m_hi, sample m values timed for the bucket)
BUCKETS = [(1, 1, (1,)), (2, 2, (2,)), (3, 4, (4,)), (5, 32, (8, 32)), (33, 256, (64, 256))]
COLD_BYTES = 300 << 20  # weight copies per shape: more than twice the 126 MB L2


def default_shapes():
    from bf16_activations_nvfp4_b200 import inputs
    shapes = list(inputs.SERVING_DECODE) + list(inputs.NARROW_N) + [inputs.SMALL_BATCH_NK, inputs.LM_HEAD_NK]
    shapes += list(inputs.QWEN36_27B_DECODE)
    seen, out = set(), []
    for s in shapes:
        if s not in seen:
            seen.add(s)
            out.append(s)
    return out


def time_tactic(fi, torch, stream, A, copies, g, out, tactic, ws) -> float:
    """Median µs per call of `tactic` over PDL-chained graph replays, every call on its own weight copy."""
    nrep = max(2, len(copies))  # one pass over the copies: every call on weights not in L2
    with torch.cuda.stream(stream):
        fi.mm_bf16_fp4(A, copies[0][0], copies[0][1], g, tactic=tactic, out=out, workspace=ws)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for r in range(nrep):
                q, s_ = copies[r % len(copies)]
                fi.mm_bf16_fp4(A, q, s_, g, tactic=tactic, out=out, workspace=ws)
        ts = []
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3 / nrep)
    del graph
    return statistics.median(ts[2:])


def tune(shapes, log=print):
    import torch

    import bf16_activations_nvfp4_b200 as fi
    from bf16_activations_nvfp4_b200 import inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    rows = []
    for n, k in shapes:
        W = torch.from_numpy(inputs.weights(n, k, seed=0)).to(dev)
        Wq, Ws, g = fi.pack_weights(W)
        del W
        wbytes = n * (k // 2 + k // 16)
        copies = [(Wq, Ws)] + [(Wq.clone(), Ws.clone()) for _ in range(-(-COLD_BYTES // wbytes) - 1)]
        for m_lo, m_hi, ms in BUCKETS:
            cands = None
            for m in ms:
                listed = set(fi.list_tactics(m, n, k))
                cands = listed if cands is None else cands & listed
            if not cands:
                continue
            A = {m: torch.from_numpy(inputs.activations(m, k, seed=0, outliers=True).view(np.int16))
                 .view(torch.bfloat16).to(dev) for m in ms}
            outs = {m: torch.empty((m, n), dtype=torch.bfloat16, device=dev) for m in ms}
            ws = torch.empty(max(max(fi.workspace_bytes(m, n, k, t) for t in cands for m in ms), 256) // 4 + 64,
                             dtype=torch.float32, device=dev)
            best = None
            for t in sorted(cands):
                total = sum(time_tactic(fi, torch, stream, A[m], copies, g, outs[m], t, ws) for m in ms)
                if best is None or total < best[1]:
                    best = (t, total)
            us = best[1] / len(ms)
            rows.append((n, k, m_lo, m_hi, sms, best[0], us))
            log(f"{n}x{k} m {m_lo}..{m_hi}: {hex(best[0])} {fi.tactic_fields(best[0])} {us:.3f} us "
                f"(mean over m = {list(ms)}; {len(cands)} candidates)")
            del ws, A, outs
        del copies, Wq, Ws, g
        torch.cuda.empty_cache()
    return rows, torch.cuda.get_device_name(dev), sms


def write_table(rows, gpu: str, sms: int, path: str = OUT) -> None:
    when = datetime.datetime.now(datetime.timezone.utc).strftime("%Y-%m-%d")
    lines = [
        "// Default-tactic table: GENERATED by bf16_activations_nvfp4_b200/tune.py; do not edit by hand.",
        f"// Measured on {gpu} ({sms} SMs), {when}: per (n, k, m bucket) the fastest tactic listed at every",
        "// sample m of the bucket, timed with cold L2 (rotating weight copies) in PDL-chained CUDA graphs.",
        "// Fields: n, k, m_lo, m_hi, SM count, tactic code, mean us per call over the bucket's sample m.",
        "static const TunedTactic kTunedTactics[] = {",
    ]
    for n, k, m_lo, m_hi, s, t, us in rows:
        lines.append(f"    {{{n}, {k}, {m_lo}, {m_hi}, {s}, 0x{t:x}, {us:.3f}}},")
    lines.append("};")
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--shapes", default=None, help="comma-separated n x k list (default: the measured workloads)")
    ap.add_argument("--out", default=OUT)
    args = ap.parse_args(argv)
    sys.path.insert(0, ROOT)
    shapes = ([tuple(int(v) for v in s.split("x")) for s in args.shapes.split(",")] if args.shapes
              else default_shapes())
    rows, gpu, sms = tune(shapes)
    write_table(rows, gpu, sms, args.out)
    print(f"wrote {len(rows)} entries to {args.out}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
