"""Pins for the oracle's quantiser, dequantiser, matmul and split-K reduce.

Checks against the hand-worked fixture, exact rational arithmetic (fractions.Fraction)
with decoders taken from the spec table and from torch, the rounding-error bound of the
quantiser, exact cases with power-of-two scales, and symmetry / permutation invariants.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bf16_activations_nvfp4_b200 import inputs
from tests._golden import code_table, hand_case

E2M1 = code_table("e2m1_values.txt")


def _e4m3_torch(code):
    return float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64))


def _unpack_codes(Wq):
    lo = Wq & 0x0F
    hi = Wq >> 4
    out = np.empty((Wq.shape[0], Wq.shape[1] * 2), np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def _bf16_value(bits):
    return float(np.array([bits], np.uint32).__lshift__(16).view(np.float32)[0])


# ------------------------------------------------------------------ hand case

def _hand_W():
    W = np.zeros((2, 16), np.float32)
    W[0] = 7 * np.array([0.5, 1, 1.5, 2, 3, 4, 6, 0, -0.5, -1, -1.5, -2, -3, -4, -6, 0])
    W[1] = 7.0
    return W


def test_hand_case_pack():
    h = hand_case()
    Wq, Ws, g = oracle.pack(_hand_W())
    assert g == np.float32(h["gscale"])
    assert Ws[0, 0] == h["scale"][0] and Ws[1, 0] == h["scale"][1]
    codes = _unpack_codes(Wq)
    assert codes[0].tolist() == h["codes"][0]
    assert codes[1].tolist() == h["codes"][1]


def test_hand_case_mm():
    h = hand_case()
    Wq, Ws, g = oracle.pack(_hand_W())
    A1 = inputs.to_bf16_bits(np.array([[1.0] * 8 + [0.0] * 8], np.float32))
    A2 = inputs.to_bf16_bits(np.ones((1, 16), np.float32))
    assert oracle.mm(A1, Wq, Ws, g)[0].tolist() == h["out"]["A_first8"]
    assert oracle.mm(A2, Wq, Ws, g)[0].tolist() == h["out"]["A_all"]


# ------------------------------------------------------- exact rational brute force

def _exact_mm(A_bits, Wq, Ws, g):
    """Independent dequant-then-dot in exact rationals (spec table + torch E4M3)."""
    codes = _unpack_codes(Wq)
    m, k = A_bits.shape
    n = Wq.shape[0]
    G = Fraction(float(g))
    out = [[Fraction(0)] * n for _ in range(m)]
    for r in range(m):
        for j in range(n):
            s = Fraction(0)
            for i in range(k):
                w = Fraction(E2M1[int(codes[j, i])]) * Fraction(_e4m3_torch(int(Ws[j, i // 16]))) * G
                s += Fraction(_bf16_value(int(A_bits[r, i]))) * w
            out[r][j] = s
    return out


@pytest.mark.parametrize("m,n,k,seed", [(1, 1, 16, 0), (2, 3, 16, 1), (3, 2, 32, 2), (3, 3, 32, 3)])
def test_mm_matches_exact_rationals(m, n, k, seed):
    A = inputs.activations(m, k, seed, outliers=(seed % 2 == 1))
    W = inputs.weights(n, k, seed, jitter=(seed >= 2))
    Wq, Ws, g = oracle.pack(W)
    ref = oracle.mm(A, Wq, Ws, g)
    exact = _exact_mm(A, Wq, Ws, g)
    for r in range(m):
        for j in range(n):
            e = exact[r][j]
            # fp64 accumulation bound: k * 2^-53 * sum |terms| (terms are exact in fp64)
            bound = k * 2.0 ** -52 * float(sum(abs(Fraction(_bf16_value(int(A[r, i])))) for i in range(k))) * 6 * 448 * float(g)
            assert abs(ref[r, j] - float(e)) <= bound, (r, j)


def test_dequant_matches_exact_decode():
    W = inputs.weights(4, 64, seed=5, jitter=True)
    Wq, Ws, g = oracle.pack(W)
    D = oracle.dequant(Wq, Ws, g)
    codes = _unpack_codes(Wq)
    for j in range(4):
        for i in range(64):
            want = E2M1[int(codes[j, i])] * _e4m3_torch(int(Ws[j, i // 16])) * float(g)
            assert D[j, i] == want


# ------------------------------------------------------------- quantiser bounds

def test_global_scale_is_amax_over_2688():
    W = inputs.weights(16, 256, seed=3)
    g = oracle.global_scale(W)
    amax = np.float32(np.max(np.abs(W)))
    assert g == np.float32(amax / np.float32(2688.0))
    assert abs(float(g) * 2688 - float(amax)) <= float(amax) * 2.0 ** -23


def test_quantisation_error_within_half_step():
    """Every element is within half an E2M1 step (times its block's denominator) of its
    dequantised value, unless it saturates at 6 * denominator; the scale is the E4M3
    rounding of (block amax / 6) / gscale."""
    W = inputs.weights(32, 512, seed=11, jitter=True)
    Wq, Ws, g = oracle.pack(W)
    D = oracle.dequant(Wq, Ws, g)
    steps = {0.0: 0.5, 0.5: 0.5, 1.0: 0.5, 1.5: 0.5, 2.0: 1.0, 3.0: 1.0, 4.0: 2.0, 6.0: 2.0}
    for j in range(32):
        for b in range(512 // 16):
            blk = W[j, b * 16:(b + 1) * 16]
            sf = _e4m3_torch(int(Ws[j, b]))
            bmax = np.float32(np.max(np.abs(blk)))
            t = np.float32(bmax / np.float32(6.0))
            want_sf = torch.tensor([float(t / g)], dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).item()
            assert sf == want_sf
            denom = float(np.float32(np.float32(sf) * g))
            for i in range(16):
                x = float(blk[i])
                d = D[j, b * 16 + i]
                mag = abs(d) / (sf * float(g)) if sf else 0.0
                if abs(x) > 6 * denom:
                    assert mag == 6.0
                else:
                    # spacing of the E2M1 grid around the chosen value
                    assert abs(x - d) <= 0.5 * steps[mag] * denom * (1 + 1e-6) + 1e-30, (j, b, i)
                if d != 0:
                    assert math.copysign(1, d) == math.copysign(1, x)


def test_pack_is_exact_on_representable_weights():
    """W = e2m1 value * sf * 2^-9 per block, with a block maximum of 6 * sf * 2^-9 and one
    block at sf = 448, so the tensor amax is 5.25 and gscale = 5.25 / 2688 = 2^-9 exactly.
    Every division in the recipe is then exact: the scales come back as the chosen E4M3
    codes, the codes as the chosen E2M1 codes, and dequant(pack(W)) == W."""
    rng = np.random.default_rng(4)
    n, k = 8, 64
    g = 2.0 ** -9
    W = np.zeros((n, k), np.float32)
    want_sf = rng.integers(0x08, 0x7F, (n, k // 16))  # normal, finite E4M3 codes
    want_sf[3, 2] = 0x7E  # 448: sets the tensor amax to 6 * 448 * 2^-9 = 5.25
    want_codes = rng.integers(0, 16, (n, k)).astype(np.uint8)
    for j in range(n):
        for b in range(k // 16):
            want_codes[j, b * 16 + int(rng.integers(0, 16))] = 7  # block max 6 * sf
            sf = _e4m3_torch(int(want_sf[j, b]))
            for i in range(16):
                W[j, b * 16 + i] = E2M1[int(want_codes[j, b * 16 + i])] * sf * g
    Wq, Ws, gs = oracle.pack(W)
    assert gs == np.float32(g)
    assert np.array_equal(Ws, want_sf.astype(np.uint8))
    got_codes = _unpack_codes(Wq)
    # -0 (code 8) stays -0: compare codes exactly
    assert np.array_equal(got_codes, want_codes)
    assert np.array_equal(oracle.dequant(Wq, Ws, gs), W.astype(np.float64))


def test_power_of_two_scaling_invariance():
    W = inputs.weights(8, 128, seed=6, jitter=True)
    Wq, Ws, g = oracle.pack(W)
    for e in (-3, 1, 4):
        Wq2, Ws2, g2 = oracle.pack(W * np.float32(2.0 ** e))
        assert np.array_equal(Wq, Wq2) and np.array_equal(Ws, Ws2)
        assert g2 == np.float32(g * np.float32(2.0 ** e))


def test_negation_symmetry():
    W = inputs.weights(8, 128, seed=12)
    A = inputs.activations(2, 128, seed=12)
    Wq, Ws, g = oracle.pack(W)
    Wq2, Ws2, g2 = oracle.pack(-W)
    assert np.array_equal(Ws, Ws2) and g == g2
    assert np.array_equal(Wq ^ 0x88, Wq2)
    assert np.array_equal(oracle.mm(A, Wq, Ws, g), -oracle.mm(A, Wq2, Ws2, g2))


def test_zero_tensor_packs_to_zero():
    W = np.zeros((3, 32), np.float32)
    Wq, Ws, g = oracle.pack(W)
    assert g == 0 and not Wq.any() and not Ws.any()
    A = inputs.activations(2, 32, seed=1)
    assert not oracle.mm(A, Wq, Ws, g).any()


def test_zero_block_gets_zero_codes():
    W = inputs.weights(2, 64, seed=2)
    W[1, 16:32] = 0.0
    Wq, Ws, g = oracle.pack(W)
    assert Ws[1, 1] == 0 and not Wq[1, 8:16].any()


# ------------------------------------------------------------- matmul structure

def test_mm_one_hot_rows_select_activation_columns():
    """W[j, perm[j]] = 5.25, else 0: gscale = 5.25/2688 = 2^-9, block scale 448, codes 6.0,
    so dequant is exactly 5.25 and out[r, j] = 5.25 * A[r, perm[j]] exactly. A transposed
    operand, a wrong index or a dropped term fails this."""
    n, k, m = 12, 48, 3
    perm = np.random.default_rng(0).permutation(k)[:n]
    W = np.zeros((n, k), np.float32)
    W[np.arange(n), perm] = 5.25
    Wq, Ws, g = oracle.pack(W)
    assert g == np.float32(2.0 ** -9)
    A = inputs.activations(m, k, seed=3)
    Af = (A.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = oracle.mm(A, Wq, Ws, g)
    assert np.array_equal(ref, 5.25 * Af[:, perm])


def test_mm_column_subset_matches_full():
    W = inputs.weights(40, 256, seed=9)
    A = inputs.activations(2, 256, seed=9)
    Wq, Ws, g = oracle.pack(W)
    full = oracle.mm(A, Wq, Ws, g)
    cols = np.array([39, 0, 17, 17, 5])
    assert np.array_equal(oracle.mm(A, Wq, Ws, g, cols=cols), full[:, cols])


def test_mm_close_to_unquantised_product():
    """Sanity: NVFP4 error on N(0, 0.02) weights is a few percent of the output rms."""
    W = inputs.weights(64, 1024, seed=1)
    A = inputs.activations(2, 1024, seed=1)
    Wq, Ws, g = oracle.pack(W)
    ref = oracle.mm(A, Wq, Ws, g)
    Af = (A.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact = Af @ W.astype(np.float64).T
    rel = np.sqrt(np.mean((ref - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    assert rel < 0.12


# ----------------------------------------------------------------- split-K reduce

def test_splitk_reduce_fixed_order():
    """((p0 + p1) + p2) in fp32: 2^24 + 1 rounds back to 2^24, so the sum is 0; any other
    order (or a wider accumulator) gives 1."""
    p = np.array([[[2.0 ** 24]], [[1.0]], [[-(2.0 ** 24)]]], np.float32)
    assert oracle.splitk_reduce(p, 1.0)[0, 0] == 0
    q = np.array([[[2.0 ** 24]], [[-(2.0 ** 24)]], [[1.0]]], np.float32)
    assert oracle.splitk_reduce(q, 1.0)[0, 0] == 0x3F80  # bf16(1.0)


def test_splitk_reduce_single_split_is_scaled_rounding():
    rng = np.random.default_rng(3)
    p = rng.standard_normal((1, 4, 33)).astype(np.float32) * 100
    g = np.float32(2.0 ** -7) * np.float32(1.5)
    ref = torch.from_numpy(p[0] * g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.splitk_reduce(p, g), ref)


def test_splitk_reduce_integer_partials_exact():
    rng = np.random.default_rng(4)
    p = rng.integers(-20, 20, (5, 3, 7)).astype(np.float32)
    got = oracle.splitk_reduce(p, 1.0)
    want = p.sum(0)
    assert np.array_equal((got.astype(np.uint32) << 16).view(np.float32), want)


def test_tolerance_helper():
    ref = np.array([[1.0, -2.0, 0.0, 4.0]])
    rms = math.sqrt((1 + 4 + 0 + 16) / 4)
    ok = oracle.within_tolerance(ref + 0.01 * np.abs(ref) + 0.0099 * rms, ref)
    assert ok.all()
    assert not oracle.within_tolerance(ref + 0.02 * np.abs(ref) + 0.011 * rms, ref).all()
