"""GPU tensor-core path (MMA tactics: TMA + tcgen05 + TMEM) against the oracle.

Tolerance for bf16 outputs: |out - ref| <= 1e-2*|ref| + 1e-2*rms(ref row), ref the oracle's
unrounded fp64 result. Exact cases (small-integer activations, weights with power-of-two
scales) must match bit for bit; the path must be bitwise deterministic over 10 reruns, and a
row's bits must not depend on m (an output element depends only on its weight row and its
activation row).
"""
import numpy as np
import pytest
import torch

import bf16_activations_nvfp4_b200 as fi
import oracle
from bf16_activations_nvfp4_b200 import inputs
from tests import _gpu
from tests.test_gpu_mm import _exact_case

pytestmark = pytest.mark.gpu

MMA = fi.make_tactic(fi.KIND_MMA, 1, 0, 0)


def _mm(A_bits, dev_w, tactic=MMA):
    Wq, Ws, g = dev_w
    out = fi.mm_bf16_fp4(_gpu.dev_bf16(A_bits), Wq, Ws, g, tactic=tactic)
    torch.cuda.synchronize()
    return _gpu.host_bits(out)


@pytest.mark.parametrize("m,n,k,seed", [(64, 512, 512, 1), (33, 300, 2048, 2), (100, 1000, 1024, 3),
                                        (256, 768, 4096, 4), (1, 256, 512, 5), (17, 257, 320, 6),
                                        (128, 4096, 1024, 7), (40, 200, 128, 13)])
def test_parity_against_oracle(m, n, k, seed):
    A = inputs.activations(m, k, seed=seed, outliers=True)
    W, (Wq, Ws, g) = _gpu.weights(n, k, seed)
    ref = oracle.mm(A, Wq, Ws, g)
    _gpu.assert_within_tolerance(_mm(A, _gpu.device_weights(n, k, seed)), ref, f"MMA {m}x{n}x{k}")


def test_default_table_takes_mma_for_larger_m():
    info = fi.resolve_tactic(64, 4096, 14336, fi.TACTIC_DEFAULT)
    assert info["kind"] == fi.KIND_MMA
    m, n, k = 64, 1000, 2048
    A = inputs.activations(m, k, seed=8)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 8)
    ref = oracle.mm(A, Wq, Ws, g)
    _gpu.assert_within_tolerance(_mm(A, _gpu.device_weights(n, k, 8), fi.TACTIC_DEFAULT), ref, "default m=64")


@pytest.mark.parametrize("m,n,k", [(40, 300, 512), (256, 512, 1024)])
def test_integer_exact_bitwise(m, n, k):
    """Small-integer activations and weights whose block scales and tensor scale are powers of
    two: every product and partial sum is exact in fp32, so the bf16 output must be the
    correctly rounded exact result bit for bit (the same case as the GEMV's)."""
    A, W = _exact_case(m, n, k, seed=m + n)
    Wq, Ws, g = oracle.pack(W)
    ref = oracle.mm(A, Wq, Ws, g)
    assert np.array_equal(ref.astype(np.float32).astype(np.float64), ref)  # exact in fp32
    want = np.array([[oracle.f32_to_bf16_bits(v) for v in row] for row in ref.astype(np.float32)], np.uint16)
    got = _mm(A, fi.pack_weights(torch.from_numpy(W).cuda()))
    assert np.array_equal(got, want)


def test_determinism_ten_reruns():
    m, n, k = 96, 1024, 2048
    A = inputs.activations(m, k, seed=9, outliers=True)
    dw = _gpu.device_weights(n, k, 9)
    base = _mm(A, dw)
    for _ in range(10):
        assert np.array_equal(_mm(A, dw), base)


def test_rows_do_not_depend_on_m():
    """Row r of the output has the same bits whether it is computed with m = 33, 64, 128 or
    256 rows (the MMA's N dimension changes with m)."""
    n, k = 768, 1024
    A256 = inputs.activations(256, k, seed=10, outliers=True)
    dw = _gpu.device_weights(n, k, 10)
    base = _mm(A256, dw)
    for m in (1, 16, 33, 64, 128, 200):
        assert np.array_equal(_mm(A256[:m], dw), base[:m]), m


def test_k_not_multiple_of_64_is_refused():
    m, n, k = 64, 256, 96
    with pytest.raises(fi.FiError) as e:
        fi.resolve_tactic(m, n, k, MMA)
    assert e.value.status == -2


@pytest.mark.parametrize("variant", [1, 2])
def test_stalled_producer_reports_timeout_and_recovers(variant):
    """Both activation modes (1: prepass conversion, 2: converted in the kernel): with the
    producers issuing nothing, every wait runs out, the error word is set, and the next call is
    correct."""
    m, n, k = 64, 512, 1024
    t = fi.make_tactic(fi.KIND_MMA, 1, 0, variant)
    assert fi.resolve_tactic(m, n, k, t)["variant"] == variant
    A = inputs.activations(m, k, seed=12)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 12)
    ref = oracle.mm(A, Wq, Ws, g)
    dw = _gpu.device_weights(n, k, 12)
    assert fi.get_device_error() == 0
    fi.debug_set(fi.DEBUG_WAIT_TIMEOUT_NS, 20_000_000)
    fi.debug_set(fi.DEBUG_STALL_PRODUCER, 1)
    try:
        _mm(A, dw, t)
        code = fi.get_device_error()
        assert code != 0, code
        assert fi.get_device_error() == 0
    finally:
        fi.debug_set(fi.DEBUG_STALL_PRODUCER, 0)
        fi.debug_set(fi.DEBUG_WAIT_TIMEOUT_NS, 1_000_000_000)
    _gpu.assert_within_tolerance(_mm(A, dw, t), ref, "after recovery")
    assert fi.get_device_error() == 0


def _split_skewed_activations(m, k, seed):
    """Activations whose K splits have very different ranges: outliers, one row scaled by 2^40 in
    its first 64 k only, one row zero over its second half, one row of tiny values."""
    A = inputs.activations_f32(m, k, seed=seed, outliers=True)
    A[0, :64] *= np.float32(2.0 ** 40)
    if m > 1:
        A[1, k // 2:] = 0.0
    if m > 2:
        A[2] *= np.float32(2.0 ** -100)
    return inputs.to_bf16_bits(A)


@pytest.mark.parametrize("m,n,k,S", [(1, 256, 512, 1), (8, 1000, 2048, 3), (17, 257, 320, 1), (40, 300, 4096, 0),
                                     (100, 1000, 1024, 2), (128, 768, 1024, 16), (16, 4096, 6144, 1)])
def test_resident_and_prepass_activations_give_the_same_bits(m, n, k, S):
    """Variant 2 converts each split's activations in the kernel's decode warps (shared memory),
    variant 1 in a prepass kernel (workspace); both scale per (row, split) with the same
    arithmetic, so outputs (bf16 and f16) are identical bit for bit, and within the oracle's
    tolerance."""
    A = _split_skewed_activations(m, k, seed=m + k)
    W, (Wq, Ws, g) = _gpu.weights(n, k, m + 3)
    dw = _gpu.device_weights(n, k, m + 3)
    res, pre = fi.make_tactic(fi.KIND_MMA, S, 0, 2), fi.make_tactic(fi.KIND_MMA, S, 0, 1)
    assert fi.resolve_tactic(m, n, k, res)["splits"] == fi.resolve_tactic(m, n, k, pre)["splits"]
    got_res = _mm(A, dw, res)
    assert np.array_equal(got_res, _mm(A, dw, pre))
    Wq_d, Ws_d, g_d = dw
    a = _gpu.dev_bf16(A)
    f16 = [fi.mm_bf16_fp4(a, Wq_d, Ws_d, g_d, tactic=t, out_dtype=torch.float16) for t in (res, pre)]
    torch.cuda.synchronize()
    assert torch.equal(f16[0], f16[1])
    ref = oracle.mm(A, Wq, Ws, g)
    _gpu.assert_within_tolerance(got_res, ref, f"resident {m}x{n}x{k} S={S}")


@pytest.mark.parametrize("m,n,k,S", [(8, 1000, 2048, 3), (40, 300, 4096, 0), (1, 256, 512, 2), (128, 768, 1024, 16)])
def test_split_k_parity(m, n, k, S):
    """K split over grid.y: fp32 partials per split, summed in split order by the reduce kernel
    (S = 0: the device-sized split)."""
    A = inputs.activations(m, k, seed=m + S, outliers=True)
    W, (Wq, Ws, g) = _gpu.weights(n, k, m + S)
    ref = oracle.mm(A, Wq, Ws, g)
    t = fi.make_tactic(fi.KIND_MMA, S, 0, 0)
    _gpu.assert_within_tolerance(_mm(A, _gpu.device_weights(n, k, m + S), t), ref, f"MMA S={S} {m}x{n}x{k}")


def test_split_k_exact_determinism_and_rows_independent_of_m():
    n, k, S = 512, 2048, 4
    t = fi.make_tactic(fi.KIND_MMA, S, 0, 0)
    A, W = _exact_case(64, n, k, seed=5)
    Wq, Ws, g = oracle.pack(W)
    ref = oracle.mm(A, Wq, Ws, g)
    want = np.array([[oracle.f32_to_bf16_bits(v) for v in row] for row in ref.astype(np.float32)], np.uint16)
    dw = fi.pack_weights(torch.from_numpy(W).cuda())
    assert np.array_equal(_mm(A, dw, t), want)
    A2 = inputs.activations(200, k, seed=6, outliers=True)
    dw2 = _gpu.device_weights(n, k, 6)
    base = _mm(A2, dw2, t)
    for _ in range(5):
        assert np.array_equal(_mm(A2, dw2, t), base)
    for m in (1, 17, 64, 128):
        assert np.array_equal(_mm(A2[:m], dw2, t), base[:m]), m


@pytest.mark.slow
@pytest.mark.parametrize("m", [64, 256])
def test_lm_head_default_sampled(m):
    """The lm_head-like GEMM at full size in the launch configuration the bench times (default
    tactic: the tensor-core path), against the oracle on every 97th column."""
    n, k = inputs.LM_HEAD_NK
    A = inputs.activations(m, k, seed=0)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 0, True)
    got = _mm(A, _gpu.device_weights(n, k, 0, True), fi.TACTIC_DEFAULT)
    cols = np.concatenate([np.arange(0, n, 97), [n - 1]])
    ref = oracle.mm(A, Wq, Ws, g, cols=cols)
    _gpu.assert_within_tolerance(got[:, cols], ref, f"lm_head m={m} (every 97th column)")


@pytest.mark.parametrize("m", [8, 32])
def test_small_batch_default_full_size_sampled(m):
    """4096 x 14336 at m = 8 and 32 (the small-batch sweep) with the default tactic, which takes
    the split-K tensor-core path there; every 13th column against the oracle."""
    n, k = inputs.SMALL_BATCH_NK
    A = inputs.activations(m, k, seed=1, outliers=True)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 1)
    got = _mm(A, _gpu.device_weights(n, k, 1), fi.TACTIC_DEFAULT)
    cols = np.concatenate([np.arange(0, n, 13), [n - 1]])
    ref = oracle.mm(A, Wq, Ws, g, cols=cols)
    _gpu.assert_within_tolerance(got[:, cols], ref, f"4096x14336 m={m}")
