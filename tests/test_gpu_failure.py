"""Failure detection on the GPU without a fault: a pipeline wait that runs out.

The test hook stalls the producer warp of the GEMV's ring pipeline for one launch, so the
consumer warps' waits on the shared-memory pipeline run out after a short limit. (The stream
pipeline has no waits between warps: each thread waits only for its own copies.) The kernel
must then end on its own, record the timeout in the device error word that the host reads,
and leave the context usable: the next call runs normally and is correct.
"""
import numpy as np
import pytest
import torch

import bf16_activations_nvfp4_b200 as fi
import oracle
from bf16_activations_nvfp4_b200 import inputs
from tests import _gpu

pytestmark = pytest.mark.gpu

RING = fi.make_tactic(fi.KIND_GEMV, 1, 0, 0x22)  # ring pipeline, two rows per stage


def test_stalled_pipeline_reports_timeout_and_recovers():
    m, n, k = 1, 1024, 4096
    A_bits = inputs.activations(m, k, seed=4)
    W, (Wq_o, Ws_o, g_o) = _gpu.weights(n, k, 4)
    ref = oracle.mm(A_bits, Wq_o, Ws_o, g_o)
    Wq, Ws, g = _gpu.device_weights(n, k, 4)
    A = _gpu.dev_bf16(A_bits)
    assert fi.get_device_error() == 0
    fi.debug_set(fi.DEBUG_WAIT_TIMEOUT_NS, 20_000_000)  # 20 ms
    fi.debug_set(fi.DEBUG_STALL_PRODUCER, 1)
    try:
        fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=RING)
        torch.cuda.synchronize()
        code = fi.get_device_error()
        assert code & 1, code  # a consumer wait ran out
        assert fi.get_device_error() == 0  # read clears it
    finally:
        fi.debug_set(fi.DEBUG_STALL_PRODUCER, 0)
        fi.debug_set(fi.DEBUG_WAIT_TIMEOUT_NS, 1_000_000_000)
    out = fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=RING)
    torch.cuda.synchronize()
    _gpu.assert_within_tolerance(_gpu.host_bits(out), ref, "after recovery")
    assert fi.get_device_error() == 0

