"""fi_mm_bf16_fp4_noalloc, the entry point for callers that may not allocate GPU memory.

An operator plugin running inside an engine that has already reserved the device's memory
(or any caller with a memory plan fixed at start-up) cannot let the library cudaMalloc a
split-K workspace, and may own no buffer to lend it either. fi_mm_bf16_fp4_noalloc keeps the
split-K partials in a static device array of the library instead. These tests call it
through the C ABI and hold it to the allocating entry point, fi_mm_bf16_fp4: two split-K
calls in a row (the second with another shape, over the partials the first one left
behind) must give exactly the bits of the allocating call with the same tactic (both run the
same kernels; only where the partials live differs), and a call whose partials would not fit
the array must be refused before anything is launched.

This file sorts last so that a run which stops at the first failure has run every other
test first; it passes on its own in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import bf16_activations_nvfp4_b200 as fi
import oracle
from bf16_activations_nvfp4_b200 import inputs
from tests import _gpu

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20  # FI_NOALLOC_SCRATCH_BYTES


def _noalloc(A, Wq, Ws, g, out, tactic):
    m, k = A.shape
    n = Wq.shape[0]
    lib = fi.library()
    return lib.fi_mm_bf16_fp4_noalloc(A.data_ptr(), Wq.data_ptr(), Ws.data_ptr(), g.data_ptr(), out.data_ptr(),
                                      m, n, k, tactic, torch.cuda.current_stream().cuda_stream)


def _allocating(A, Wq, Ws, g, tactic):
    m, k = A.shape
    n = Wq.shape[0]
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    st = fi.library().fi_mm_bf16_fp4(A.data_ptr(), Wq.data_ptr(), Ws.data_ptr(), g.data_ptr(), out.data_ptr(),
                                     m, n, k, tactic, torch.cuda.current_stream().cuda_stream)
    assert st == 0, fi.last_error()
    return out


@pytest.mark.parametrize("splits", [4, 8])
def test_two_calls_in_a_row_match_the_allocating_entry_point(splits):
    tactic = fi.make_tactic(fi.KIND_GEMV, splits, 0, 0)
    calls = [(3, 1000, 4096, 11), (2, 600, 2048, 12)]  # ragged n; the second reuses dirty scratch
    for m, n, k, seed in calls:
        assert 0 < fi.workspace_bytes(m, n, k, tactic) <= SCRATCH_BYTES
        A = _gpu.dev_bf16(inputs.activations(m, k, seed=seed))
        Wq, Ws, g = _gpu.device_weights(n, k, seed)
        out = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = _noalloc(A, Wq, Ws, g, out, tactic)
        assert st == 0, fi.last_error()
        ref = _allocating(A, Wq, Ws, g, tactic)
        torch.cuda.synchronize()
        assert np.array_equal(_gpu.host_bits(out), _gpu.host_bits(ref)), f"m={m} n={n} k={k} S={splits}"


def test_single_split_needs_no_scratch():
    m, n, k = 1, 512, 2048
    tactic = fi.make_tactic(fi.KIND_GEMV, 1, 0, 0)
    A = _gpu.dev_bf16(inputs.activations(m, k, seed=3))
    Wq, Ws, g = _gpu.device_weights(n, k, 0)
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(A, Wq, Ws, g, out, tactic) == 0, fi.last_error()
    ref = _allocating(A, Wq, Ws, g, tactic)
    torch.cuda.synchronize()
    assert np.array_equal(_gpu.host_bits(out), _gpu.host_bits(ref)), "single split"


def test_partials_beyond_the_static_scratch_are_refused():
    m, n, k = 32, 8192, 4096
    tactic = fi.make_tactic(fi.KIND_GEMV, 8, 0, 0)
    assert fi.workspace_bytes(m, n, k, tactic) > SCRATCH_BYTES
    A = _gpu.dev_bf16(inputs.activations(m, k, seed=5))
    Wq = torch.zeros((n, k // 2), dtype=torch.uint8, device="cuda")
    Ws = torch.zeros((n, k // 16), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, dtype=torch.float32, device="cuda")
    out = torch.full((m, n), 7.0, dtype=torch.bfloat16, device="cuda")
    st = _noalloc(A, Wq, Ws, g, out, tactic)
    assert st == -4  # FI_ERR_WORKSPACE
    assert "scratch" in fi.last_error()
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was launched


def test_default_tactic_falls_back_to_a_split_that_fits():
    """5120 x 17408 (a Qwen3.6-27B down projection) at m = 32: the default (the tensor-core path
    with 7 K splits) needs more scratch than the static array holds; the allocation-free entry
    point takes the largest smaller split that fits and stays within tolerance."""
    m, n, k = 32, 5120, 17408
    assert fi.workspace_bytes(m, n, k) > 4 << 20
    A_bits = inputs.activations(m, k, seed=3)
    W, (Wq_o, Ws_o, g_o) = _gpu.weights(n, k, 3)
    dw = _gpu.device_weights(n, k, 3)
    cols = np.concatenate([np.arange(0, n, 31), [n - 1]])
    ref = oracle.mm(A_bits, Wq_o, Ws_o, g_o, cols=cols)
    Wq, Ws, g = dw
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    st = _noalloc(_gpu.dev_bf16(A_bits), Wq, Ws, g, out, fi.TACTIC_DEFAULT)
    assert st == 0, fi.last_error()
    torch.cuda.synchronize()
    _gpu.assert_within_tolerance(_gpu.host_bits(out)[:, cols], ref, "no-alloc default, m=32")


def test_default_falls_back_to_a_single_split_gemv():
    """150016 x 5120 at m = 4 (a shape the generated tactic table does not list, so the built-in
    rules decide): the default (GEMV with two K splits) needs about 4.8 MB of partials; the only
    smaller split, S = 1, needs no scratch at all and must be the one taken. Its bits equal the
    allocating call's with that tactic, and it stays within tolerance of the oracle on sampled
    columns."""
    m, n, k = 4, 150016, 5120
    info = fi.resolve_tactic(m, n, k, fi.TACTIC_DEFAULT)
    assert info["kind"] == fi.KIND_GEMV and info["splits"] > 1 and info["workspace_bytes"] > SCRATCH_BYTES
    fallback = fi.make_tactic(fi.KIND_GEMV, 1, 0, 0)  # the automatic pipeline: any S = 1 GEMV gives these bits
    fb = fi.resolve_tactic(m, n, k, fallback)
    assert fb["splits"] == 1 and fb["workspace_bytes"] == 0
    A_bits = inputs.activations(m, k, seed=4)
    W, (Wq_o, Ws_o, g_o) = _gpu.weights(n, k, 0, True)
    Wq, Ws, g = _gpu.device_weights(n, k, 0, True)
    A = _gpu.dev_bf16(A_bits)
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    st = _noalloc(A, Wq, Ws, g, out, fi.TACTIC_DEFAULT)
    assert st == 0, fi.last_error()
    ref = _allocating(A, Wq, Ws, g, fallback)
    torch.cuda.synchronize()
    got = _gpu.host_bits(out)
    assert np.array_equal(got, _gpu.host_bits(ref))
    cols = np.concatenate([np.arange(0, n, 499), [n - 1]])
    _gpu.assert_within_tolerance(got[:, cols], oracle.mm(A_bits, Wq_o, Ws_o, g_o, cols=cols), "no-alloc m=4 lm_head")
