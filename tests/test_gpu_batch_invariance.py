"""Batch invariance and run-to-run determinism of every tactic on the small-batch workload.

Workload: n x k = 4096 x 14336, activations N(0,1) in bf16 with 1% of the entries scaled by
50 (outliers), m in {1, 2, 4, 8, 16, 32}. For every tactic code that fi_list_tactics offers at
any of these m (GEMV and MMA, splits 1, 2, 4, 8 and device-sized, every pipeline), the rows
of the output must be bitwise the same at every m where the code resolves, over 10 reruns
each: the batch-invariant property the FlashInfer v0.7.4 article describes for its GEMMs (a
row's bits do not depend on how many rows share the call), and the fixed-order split-K of
PR #4038 ("What it does", the split-K item).
"""
import numpy as np
import pytest
import torch

import bf16_activations_nvfp4_b200 as fi
from bf16_activations_nvfp4_b200 import inputs
from tests import _gpu

pytestmark = pytest.mark.gpu

MS = [1, 2, 4, 8, 16, 32]
RERUNS = 10


def _run(A, dw, tactic, out):
    Wq, Ws, g = dw
    fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=tactic, out=out)


def _tactics_by_m(n, k):
    """{tactic code: [m where it resolves]} over the codes listed at any m of the sweep."""
    codes = []
    for m in MS:
        for t in fi.list_tactics(m, n, k):
            if t not in codes:
                codes.append(t)
    table = {}
    for t in codes:
        ok = []
        for m in MS:
            try:
                fi.resolve_tactic(m, n, k, t)
                ok.append(m)
            except fi.FiError:
                pass
        if ok:
            table[t] = ok
    return table


def _check(n, k, table):
    A_all = _gpu.dev_bf16(inputs.activations(MS[-1], k, seed=0, outliers=True))
    dw = _gpu.device_weights(n, k, 0)
    ws = torch.empty(max(fi.workspace_bytes(m, n, k, t) for t, ms in table.items() for m in ms) // 4 + 64,
                     dtype=torch.float32, device="cuda")
    fi.set_workspace(ws)
    try:
        for t, ms in table.items():
            S = {fi.resolve_tactic(m, n, k, t)["splits"] for m in ms}
            assert len(S) == 1, (fi.tactic_fields(t), S)  # the resolved split is the same for every m
            base_out = torch.empty((ms[-1], n), dtype=torch.bfloat16, device="cuda")
            _run(A_all[:ms[-1]], dw, t, base_out)
            base = _gpu.host_bits(base_out)
            for m in ms:
                out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
                for r in range(RERUNS):
                    out.fill_(float("nan"))
                    _run(A_all[:m], dw, t, out)
                    got = _gpu.host_bits(out)
                    assert np.array_equal(got, base[:m]), (fi.tactic_fields(t), m, r)
    finally:
        fi.set_workspace(None)


def test_every_listed_tactic_is_batch_invariant_and_deterministic():
    n, k = inputs.SMALL_BATCH_NK
    table = _tactics_by_m(n, k)
    kinds = {(fi.tactic_fields(t)["kind"], fi.tactic_fields(t)["splits"]) for t in table}
    # the split menu of both kinds is covered
    for kind in (fi.KIND_GEMV, fi.KIND_MMA):
        assert {(kind, S) for S in (1, 2, 4, 8, 0)} <= kinds, kinds
    _check(n, k, table)


def test_mma_device_sized_split_rows_match_from_m1_to_m32():
    """14336 x 4096: the device-sized MMA split resolves once for every m, so row 0 at m = 1 is
    bitwise row 0 at m = 32."""
    n, k = 14336, 4096
    t = fi.make_tactic(fi.KIND_MMA, 0, 0, 0)
    _check(n, k, {t: MS})
