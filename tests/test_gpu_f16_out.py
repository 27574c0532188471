"""fp16 output (PR #4038: the commit that covers fp16 output through the GEMV path, and its
test of fp16 GEMV output), through fi_mm_bf16_fp4_out and fi_splitk_reduce_out.

The fp32 arithmetic before the final rounding is the same as for the bf16 output; the last
step rounds to IEEE binary16 instead (nearest even, +-inf from 65520 on). Checked: parity with
the oracle's unrounded fp64 result within the tolerance used for bf16 (f16 rounds finer), the
exact f16 rounding of exact results for every tactic, and the reduce bit for bit against the
oracle's definition.
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

GEMV, MMA = fi.KIND_GEMV, fi.KIND_MMA


def _f16_bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.float16
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def _f16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bits.view(np.float16).astype(np.float64)


def _mm_f16(A_bits, dw, tactic):
    Wq, Ws, g = dw
    out = fi.mm_bf16_fp4(_gpu.dev_bf16(A_bits), Wq, Ws, g, tactic=tactic, out_dtype=torch.float16)
    torch.cuda.synchronize()
    return _f16_bits(out)


@pytest.mark.parametrize("m,n,k,seed", [(1, 512, 2048, 0), (1, 1000, 2688, 1), (3, 777, 4096, 2), (64, 300, 1024, 3),
                                        (1, 4096, 14336, 4)])
def test_f16_output_parity(m, n, k, seed):
    A = inputs.activations(m, k, seed, outliers=True)
    W, (Wq, Ws, g) = _gpu.weights(n, k, seed)
    ref = oracle.mm(A, Wq, Ws, g)
    dw = _gpu.device_weights(n, k, seed)
    tactics = [fi.TACTIC_DEFAULT]
    if m <= 32:
        tactics += [fi.make_tactic(GEMV, 1, 0, 0), fi.make_tactic(GEMV, 3, 0, 0)]
    if k % 64 == 0:
        tactics += [fi.make_tactic(MMA, 1, 0, 0), fi.make_tactic(MMA, 4, 0, 0)]
    for t in tactics:
        got = _f16_to_f64(_mm_f16(A, dw, t))
        ok = oracle.within_tolerance(got, ref, _gpu.RTOL, _gpu.RRMS)
        assert ok.all(), (t, np.argwhere(~ok)[:3])


@pytest.mark.parametrize("m,n,k", [(1, 256, 1024), (4, 100, 2688), (40, 300, 512)])
def test_f16_output_of_exact_results_is_their_exact_rounding(m, n, k):
    A, W = _exact_case(m, n, k, seed=m + n + 1)
    Wq, Ws, g = oracle.pack(W)
    ref = oracle.mm(A, Wq, Ws, g)
    assert np.array_equal(ref.astype(np.float32).astype(np.float64), ref)  # exact in fp32
    want = oracle.round_out(ref.astype(np.float32), "f16")
    dw = fi.pack_weights(torch.from_numpy(W).cuda())
    for t in fi.list_tactics(m, n, k):
        assert np.array_equal(_mm_f16(A, dw, t), want), fi.tactic_fields(t)


def test_f16_and_bf16_outputs_round_one_fp32_result():
    """Both outputs of one tactic are round-to-nearest of the same fp32 value x, each within half
    an ulp of x, so |f16 - bf16| <= ulp_bf16(x)/2 + ulp_f16(x)/2 element by element (on random
    inputs, where the two roundings differ)."""
    m, n, k = 3, 700, 2048
    A = inputs.activations(m, k, seed=19, outliers=True)
    dw = _gpu.device_weights(n, k, 19)
    Wq, Ws, g = dw
    for t in (fi.make_tactic(GEMV, 1, 0, 0), fi.make_tactic(GEMV, 4, 0, 0), fi.make_tactic(MMA, 2, 0, 0)):
        f16 = _f16_to_f64(_mm_f16(A, dw, t))
        bf = fi.mm_bf16_fp4(_gpu.dev_bf16(A), Wq, Ws, g, tactic=t)
        torch.cuda.synchronize()
        bf16 = _gpu.bits_to_f64(_gpu.host_bits(bf))
        mag = np.maximum(np.abs(bf16), 2.0 ** -14)
        ulp_bf16 = np.exp2(np.floor(np.log2(mag)) - 7)
        ulp_f16 = np.exp2(np.floor(np.log2(mag)) - 10)
        assert np.all(np.abs(f16 - bf16) <= 0.5 * ulp_bf16 + 0.5 * ulp_f16 + 2.0 ** -24), fi.tactic_fields(t)
        assert not np.array_equal(f16, bf16)  # the roundings differ: the output type took effect


def test_splitk_reduce_f16_bitwise_against_definition():
    rng = np.random.default_rng(12)
    for S, m, n in [(1, 1, 7), (2, 3, 1001), (7, 2, 64), (130, 1, 515)]:
        p = (rng.standard_normal((S, m, n)) * 500).astype(np.float32)
        p[0, 0, :3] = [70000.0, -70000.0, 65519.0]  # overflow to +-inf, largest finite
        g = np.float32(1.0 if S == 1 else 0.7)
        want = oracle.splitk_reduce(p, g, "f16")
        got = fi.splitk_reduce(torch.from_numpy(p).cuda(), torch.tensor([g], device="cuda"), out_dtype=torch.float16)
        torch.cuda.synchronize()
        assert np.array_equal(_f16_bits(got), want), (S, m, n)


def test_out_dtype_is_checked():
    W, _ = _gpu.weights(8, 64, 0)
    Wq, Ws, g = fi.pack_weights(torch.from_numpy(W).cuda())
    A = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((2, 8), dtype=torch.float16, device="cuda")
    st = fi.library().fi_mm_bf16_fp4_out(A.data_ptr(), Wq.data_ptr(), Ws.data_ptr(), g.data_ptr(), out.data_ptr(),
                                         2, 2, 8, 64, fi.TACTIC_DEFAULT, None, 0,
                                         torch.cuda.current_stream().cuda_stream)
    assert st == -1
    with pytest.raises(ValueError):
        fi.mm_bf16_fp4(A, Wq, Ws, g, out_dtype=torch.float32)
