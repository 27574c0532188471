"""GPU matmul (fi_mm_bf16_fp4, fi_splitk_reduce) against the oracle.

Tolerance for bf16 outputs: |out - ref| <= 1e-2*|ref| + 1e-2*rms(ref row), with ref the
oracle's unrounded fp64 result. Exact cases (small-integer activations, weights with
power-of-two scales) must match bit for bit; every tactic must be bitwise deterministic
over 10 reruns, and for a fixed tactic row r of the output must not depend on m.
"""
import numpy as np
import pytest
import torch

import bf16_activations_nvfp4_b200 as fi
import oracle
from bf16_activations_nvfp4_b200 import inputs
from tests import _gpu

pytestmark = pytest.mark.gpu

GEMV = fi.KIND_GEMV


def _mm(A_bits, dev_w, tactic=fi.TACTIC_DEFAULT, **kw):
    Wq, Ws, g = dev_w
    out = fi.mm_bf16_fp4(_gpu.dev_bf16(A_bits), Wq, Ws, g, tactic=tactic, **kw)
    torch.cuda.synchronize()
    return _gpu.host_bits(out)


def _tactics(m, n, k):
    return fi.list_tactics(m, n, k)


# ------------------------------------------------------------- parity, small sizes

def test_tiny_workload_every_tactic():
    """m=1, n=512, k=2048, seed 0: the tiny correctness workload, every listed tactic."""
    m, n, k = 1, 512, 2048
    A = inputs.activations(m, k, seed=0)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 0)
    ref = oracle.mm(A, Wq, Ws, g)
    dw = _gpu.device_weights(n, k, 0)
    ts = _tactics(m, n, k)
    assert len(ts) >= 6
    for t in ts + [fi.TACTIC_DEFAULT]:
        _gpu.assert_within_tolerance(_mm(A, dw, t), ref, f"tactic {fi.tactic_fields(t) if t >= 0 else t}")


@pytest.mark.parametrize("m,n,k,seed", [
    (1, 1000, 2688, 1),     # ragged k tail (2688 = 2.6 warp steps), n not a multiple of 8
    (3, 777, 4096, 2),      # m not a power of two, odd n
    (8, 2048, 7168, 3),
    (5, 129, 1056, 4),      # k = 33 chunks
    (2, 1, 32, 5),          # single chunk, single row
    (16, 300, 2048, 6),
    (32, 96, 1024, 7),
    (1, 1001, 1536, 8),     # 48 chunks: a half-filled last iteration, odd n
    (4, 515, 5120, 9),      # 160 chunks: an item whose second iteration is empty, partial group
])
def test_parity_spanning_tiles(m, n, k, seed):
    A = inputs.activations(m, k, seed, outliers=True)
    W, (Wq, Ws, g) = _gpu.weights(n, k, seed, True)
    ref = oracle.mm(A, Wq, Ws, g)
    dw = _gpu.device_weights(n, k, seed, True)
    for t in _tactics(m, n, k):
        _gpu.assert_within_tolerance(_mm(A, dw, t), ref, f"m={m} n={n} k={k} {fi.tactic_fields(t)}")


def _exact_case(m, n, k, seed):
    """Small-integer activations (|a| <= 2) and weights e2m1 * 448 * 2^-j * 2^-9 with one
    block at the tensor maximum, so gscale = 2^-9 exactly and every block scale is 448 * 2^-j.
    Every product is then a multiple of 7 * 2^(5-jmax) * gscale-free units and every partial
    sum of <= k terms stays below 2^24 of those units: fp32 accumulation is exact in any
    order, so every tactic must return exactly bf16_rn(exact result)."""
    rng = np.random.default_rng(seed)
    A = inputs.to_bf16_bits(rng.integers(-2, 3, (m, k)).astype(np.float32))
    E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    W = E2M1[rng.integers(0, 8, (n, k))] * rng.choice([-1, 1], (n, k)).astype(np.float32)
    W[:, ::16] = 6.0
    e = rng.integers(-2, 1, (n, k // 16)).astype(np.float32)
    W *= np.repeat(np.exp2(e), 16, axis=1) * np.float32(448 * 2.0 ** -9)
    W[0, 0:16] = np.abs(W[0, 0:16]) / np.exp2(e[0, 0])  # block 0 at scale 448: tensor amax 5.25
    return A, W


@pytest.mark.parametrize("m,n,k", [(1, 256, 1024), (4, 100, 2688), (32, 64, 512)])
def test_integer_exact_bitwise(m, n, k):
    A, W = _exact_case(m, n, k, seed=m + n)
    Wq, Ws, g = oracle.pack(W)
    assert g == np.float32(2.0 ** -9)
    ref = oracle.mm(A, Wq, Ws, g)
    assert np.array_equal(ref.astype(np.float32).astype(np.float64), ref)  # exact in fp32
    want = np.array([[oracle.f32_to_bf16_bits(v) for v in row] for row in ref.astype(np.float32)], np.uint16)
    dw = fi.pack_weights(torch.from_numpy(W).cuda())
    for t in _tactics(m, n, k):
        got = _mm(A, dw, t)
        assert np.array_equal(got, want), fi.tactic_fields(t)


# ---------------------------------------------------------------- properties

def test_determinism_ten_reruns_every_tactic():
    m, n, k = 4, 4096, 4096
    A = inputs.activations(m, k, seed=3, outliers=True)
    dw = _gpu.device_weights(n, k, 3)
    for t in _tactics(m, n, k):
        first = _mm(A, dw, t)
        for _ in range(9):
            assert np.array_equal(_mm(A, dw, t), first), fi.tactic_fields(t)


@pytest.mark.parametrize("splits", [0, 8, 12])
def test_batch_invariance_rows_do_not_depend_on_m(splits):
    """4096 x 14336, activations with 1% x50 outliers: row 0 (and every row r < m) of a fixed
    tactic is bitwise the same for m in {1, 2, 4, 8, 16, 32}, over 10 reruns."""
    n, k = 4096, 14336
    A32 = inputs.activations(32, k, seed=0, outliers=True)
    dw = _gpu.device_weights(n, k, 0)
    ms = [1, 2, 4, 8, 16, 32]
    for R in (0, 1):  # automatic rows per stage (varies with m) and one row per stage
        t = fi.make_tactic(GEMV, splits, 0, R)
        base = _mm(A32[:ms[-1]], dw, t)
        for m in ms:
            for _ in range(10 if m in (1, ms[-1]) else 2):
                got = _mm(A32[:m], dw, t)
                assert np.array_equal(got, base[:m]), (R, splits, m)


def test_batch_invariance_many_rows_per_stage_small_m():
    n, k = 4096, 14336
    A4 = inputs.activations(4, k, seed=1, outliers=True)
    dw = _gpu.device_weights(n, k, 0)
    t = fi.make_tactic(GEMV, 8, 0, 4)
    base = _mm(A4, dw, t)
    for m in (1, 2, 3, 4):
        for _ in range(3):
            assert np.array_equal(_mm(A4[:m], dw, t), base[:m]), m


def test_rows_per_stage_and_occupancy_do_not_change_bits():
    """Only the kind and S fix the arithmetic: the pipeline, rows per warp and CTAs per SM only
    move work between warps and CTAs."""
    m, n, k = 2, 2048, 7168
    A = inputs.activations(m, k, seed=9)
    dw = _gpu.device_weights(n, k, 0)
    for S in (1, 3):
        variants = [(0x10 | R, c) for R in (0, 1, 2, 4) for c in (1, 2)] + [(0x20 | R, 1) for R in (0, 1, 8)]
        outs = [_mm(A, dw, fi.make_tactic(GEMV, S, c, v)) for v, c in variants]
        for (v, c), o in zip(variants[1:], outs[1:]):
            assert np.array_equal(o, outs[0]), (S, hex(v), c)


def test_pipelines_give_identical_bits():
    """The per-warp async-copy pipeline, the producer-warp ring, the overlapped variant, the
    register pipeline and the lean stream pipeline run the same per-chunk arithmetic in the
    same order, so for one S their outputs are bitwise equal."""
    # (1, 20000, 2048): several row groups per warp
    for m, n, k in [(1, 2048, 7168), (3, 1000, 4096), (8, 515, 2688), (32, 300, 2048), (1, 333, 4096), (1, 97, 8192),
                    (1, 20000, 2048)]:
        A = inputs.activations(m, k, seed=21, outliers=True)
        dw = _gpu.device_weights(n, k, 2)
        for S in (1, 2, 5):
            try:
                stream = _mm(A, dw, fi.make_tactic(GEMV, S, 0, 0x10))
            except fi.FiError as e:  # activations of this split do not fit half an SM
                assert e.status == -2
                continue
            for var in (0x20, 0x30, 0x40, 0x41, 0x50, 0x51, 0x52, 0x54):
                try:
                    other = _mm(A, dw, fi.make_tactic(GEMV, S, 0, var))
                except fi.FiError as e:
                    # the overlapped variant's half SM cannot hold these activations; the lean
                    # pipeline takes m = 1 with k % 256 == 0 and splits of whole items only
                    assert e.status == -2 and (var == 0x30 or var >> 4 == 5), (m, n, k, S, hex(var))
                    continue
                assert np.array_equal(stream, other), (m, n, k, S, hex(var))


@pytest.mark.parametrize("n,k", [(1000, 2688), (777, 1056), (300, 4096), (2048, 7168)])
def test_automatic_pipeline_of_split_calls_at_m1(n, k):
    """At m = 1 with S > 1 the automatic pipeline may be the register pipeline with two CTAs
    per SM (k % 256 != 0) or the stream pipeline with four rows per item: within tolerance of
    the oracle and bitwise equal to the stream pipeline with two rows per item at the same S."""
    A = inputs.activations(1, k, seed=31, outliers=True)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 4, True)
    ref = oracle.mm(A, Wq, Ws, g)
    dw = _gpu.device_weights(n, k, 4, True)
    for S in (2, 3, 8, 0):
        t = fi.make_tactic(GEMV, S, 0, 0)
        auto = _mm(A, dw, t)
        _gpu.assert_within_tolerance(auto, ref, f"n={n} k={k} S={S}")
        S_res = fi.resolve_tactic(1, n, k, t)["splits"]
        assert np.array_equal(auto, _mm(A, dw, fi.make_tactic(GEMV, S_res, 0, 0x12))), (n, k, S)


def test_multi_slab_rows_and_many_splits():
    """k = 65536 needs several ring stages per row (slabs); narrow n and ragged shapes."""
    for m, n, k, S in [(1, 8, 65536, 1), (2, 33, 16384, 5), (3, 17, 32768, 2)]:
        A = inputs.activations(m, k, seed=m + S, outliers=True)
        W, (Wq, Ws, g) = _gpu.weights(n, k, 3)
        ref = oracle.mm(A, Wq, Ws, g)
        dw = _gpu.device_weights(n, k, 3)
        for R in (0, 1):  # one 32 KB row per stage is what fits next to A at k = 65536
            _gpu.assert_within_tolerance(_mm(A, dw, fi.make_tactic(GEMV, S, 0, R)), ref, f"{m}x{n}x{k} S={S} R={R}")


def test_split_counts_agree_within_tolerance():
    m, n, k = 1, 4096, 14336
    A = inputs.activations(m, k, seed=0)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 0)
    ref = oracle.mm(A, Wq, Ws, g)
    dw = _gpu.device_weights(n, k, 0)
    for S in (1, 2, 4, 8, 16, 64):
        _gpu.assert_within_tolerance(_mm(A, dw, fi.make_tactic(GEMV, S, 0, 2)), ref, f"S={S}")


# ------------------------------------------------------------------- full sizes

@pytest.mark.parametrize("n,k", inputs.SERVING_DECODE)
def test_serving_decode_shapes_default_tactic(n, k):
    """m=1 serving decode shapes at full size, in the launch configuration the benchmark
    times (default tactic), against the full oracle product."""
    A = inputs.activations(1, k, seed=0)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 0)
    ref = oracle.mm(A, Wq, Ws, g)
    dw = _gpu.device_weights(n, k, 0)
    _gpu.assert_within_tolerance(_mm(A, dw), ref, f"{n}x{k}")
    for S in (1, 2, 4, 8):
        _gpu.assert_within_tolerance(_mm(A, dw, fi.make_tactic(GEMV, S, 0, 0)), ref, f"{n}x{k} S={S}")


@pytest.mark.parametrize("n,k", inputs.NARROW_N)
def test_narrow_n_sweep_seeds(n, k):
    for seed in range(6):
        A = inputs.activations(1, k, seed=seed)
        W, (Wq, Ws, g) = _gpu.weights(n, k, seed)
        ref = oracle.mm(A, Wq, Ws, g)
        dw = fi.pack_weights(torch.from_numpy(W).cuda())
        _gpu.assert_within_tolerance(_mm(A, dw), ref, f"{n}x{k} seed {seed}")


@pytest.mark.slow
def test_lm_head_m1_sampled():
    n, k = inputs.LM_HEAD_NK
    A = inputs.activations(1, k, seed=0)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 0, True)
    dw = _gpu.device_weights(n, k, 0, True)
    got = _mm(A, dw)
    cols = np.concatenate([np.arange(0, n, 97), [n - 1]])
    ref = oracle.mm(A, Wq, Ws, g, cols=cols)
    _gpu.assert_within_tolerance(got[:, cols], ref, "lm_head m=1 (every 97th column)")


@pytest.mark.slow
@pytest.mark.parametrize("n,k", inputs.QWEN36_27B_DECODE)
def test_qwen36_27b_decode_shapes_default_sampled(n, k):
    """The second workload (PR #4038's Qwen3.6-27B-NVFP4 decode GEMMs at m = 1, synthetic weights):
    the default tactic and two split tactics at full size, every 61st output column (and the
    last) against the oracle."""
    A = inputs.activations(1, k, seed=2)
    W, (Wq, Ws, g) = _gpu.weights(n, k, 2)
    dw = fi.pack_weights(torch.from_numpy(W).cuda())
    cols = np.concatenate([np.arange(0, n, 61), [n - 1]])
    ref = oracle.mm(A, Wq, Ws, g, cols=cols)
    for t in (fi.TACTIC_DEFAULT, fi.make_tactic(GEMV, 2, 0, 0), fi.make_tactic(GEMV, 0, 0, 0)):
        _gpu.assert_within_tolerance(_mm(A, dw, t)[:, cols], ref, f"{n}x{k} {t}")
    del dw
    torch.cuda.empty_cache()


# ------------------------------------------------------------------- split-K reduce

def test_splitk_reduce_bitwise_against_definition():
    rng = np.random.default_rng(11)
    for S, m, n in [(1, 1, 7), (2, 3, 1001), (7, 2, 64), (130, 1, 515)]:
        p = (rng.standard_normal((S, m, n)) * 50).astype(np.float32)
        g = np.float32(0.0123)
        want = oracle.splitk_reduce(p, g)
        got = fi.splitk_reduce(torch.from_numpy(p).cuda(), torch.tensor([g], device="cuda"))
        torch.cuda.synchronize()
        assert np.array_equal(_gpu.host_bits(got), want), (S, m, n)


def test_splitk_reduce_order_is_fixed():
    p = np.array([[[2.0 ** 24]], [[1.0]], [[-(2.0 ** 24)]]], np.float32)
    got = fi.splitk_reduce(torch.from_numpy(p).cuda(), torch.ones(1, device="cuda"))
    assert _gpu.host_bits(got)[0, 0] == 0


# ------------------------------------------------------------------- edge cases

def test_empty_and_zero_k():
    dw = (torch.empty((5, 0), dtype=torch.uint8, device="cuda"),
          torch.empty((5, 0), dtype=torch.uint8, device="cuda"), torch.ones(1, device="cuda"))
    A = torch.empty((3, 0), dtype=torch.bfloat16, device="cuda")
    out = torch.full((3, 5), 1.0, dtype=torch.bfloat16, device="cuda")
    fi.mm_bf16_fp4(A, *dw, out=out)
    assert not out.float().any()
    W, _ = _gpu.weights(8, 64, 0)
    Wq, Ws, g = fi.pack_weights(torch.from_numpy(W).cuda())
    out0 = fi.mm_bf16_fp4(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"), Wq, Ws, g)
    assert out0.shape == (0, 8)


def test_errors_raise():
    W, _ = _gpu.weights(8, 64, 0)
    Wq, Ws, g = fi.pack_weights(torch.from_numpy(W).cuda())
    A = torch.zeros((33, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fi.FiError) as e:
        fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=fi.make_tactic(GEMV, 1, 0, 1))
    assert e.value.status == -2
    small = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(fi.FiError) as e:
        fi.mm_bf16_fp4(A[:2], Wq, Ws, g, tactic=fi.make_tactic(GEMV, 2, 0, 1), workspace=small)
    assert e.value.status == -4


def test_workspace_registration_and_graph_capture():
    m, n, k = 2, 1024, 4096
    A = _gpu.dev_bf16(inputs.activations(m, k, seed=1))
    W, (Wq_o, Ws_o, g_o) = _gpu.weights(n, k, 1)
    ref = oracle.mm(inputs.activations(m, k, seed=1), Wq_o, Ws_o, g_o)
    Wq, Ws, g = _gpu.device_weights(n, k, 1)
    t = fi.make_tactic(GEMV, 4, 0, 1)
    eager = fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=t)
    ws = torch.empty(fi.workspace_bytes(m, n, k, t) // 4 + 64, dtype=torch.float32, device="cuda")
    fi.set_workspace(ws)
    try:
        out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=t, out=out)  # warm-up outside capture
            with torch.cuda.graph(graph, stream=s):
                fi.mm_bf16_fp4(A, Wq, Ws, g, tactic=t, out=out)
        torch.cuda.current_stream().wait_stream(s)
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
        _gpu.assert_within_tolerance(_gpu.host_bits(out), ref, "graph replay")
    finally:
        fi.set_workspace(None)
