"""Pins for the oracle's element formats (E2M1, E4M3, bf16 rounding).

Each check compares the oracle with something other than itself: the hand-written spec
tables under tests/golden/, torch's own float8_e4m3fn / bfloat16 conversions, and brute
force over the whole code space.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests._golden import code_table

E2M1 = code_table("e2m1_values.txt")


def _same(a, b):
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return a == b and math.copysign(1, a) == math.copysign(1, b)


def test_e2m1_decode_matches_spec_table():
    assert sorted(E2M1) == list(range(16))
    for c, v in E2M1.items():
        assert _same(oracle.e2m1_decode(c), v), c


def test_e4m3_decode_anchor_values():
    for c, v in code_table("e4m3_anchors.txt").items():
        assert _same(oracle.e4m3_decode(c), v), hex(c)


def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        assert _same(oracle.e4m3_decode(c), float(ref[c])), hex(c)


def test_e4m3_decode_monotone():
    vals = [oracle.e4m3_decode(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(vals, vals[1:]))


def _brute_encode(x, grid):
    """Nearest grid value (list of (value, code)), ties to the even code; saturating."""
    ax = abs(x)
    best = None
    for v, c in grid:
        d = abs(ax - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0 and best[2] % 2 == 1):
            best = (d, v, c)
    return best[2]


def _e4m3_grid():
    return [(oracle.e4m3_decode(c), c) for c in range(0x7F)]


def _e2m1_grid():
    return [(E2M1[c], c) for c in range(8)]


def _midpoints(grid):
    vals = sorted(v for v, _ in grid)
    return [(a + b) / 2 for a, b in zip(vals, vals[1:])]


def test_e4m3_encode_brute_force():
    grid = _e4m3_grid()
    rng = np.random.default_rng(7)
    xs = list(np.float32(rng.uniform(0, 500, 3000))) + list(np.float32(np.exp(rng.uniform(-14, 6.2, 3000))))
    xs += [np.float32(m) for m in _midpoints(grid)]
    for x in xs:
        x = float(x)
        want = _brute_encode(x, grid)  # argmin over finite codes; > 448 saturates to 0x7e
        assert oracle.e4m3_encode(x) == want, x
        assert oracle.e4m3_encode(-x) == want | 0x80, x


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(8)
    x = np.float32(np.exp(rng.uniform(-12, math.log(448), 20000)) * rng.choice([-1, 1], 20000))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    for x in (448.0, 460.0, 464.0, 1e6, 3.0e38):
        assert oracle.e4m3_encode(x) == 0x7E
        assert oracle.e4m3_encode(-x) == 0xFE


def test_e2m1_encode_brute_force_and_midpoints():
    grid = _e2m1_grid()
    rng = np.random.default_rng(9)
    xs = list(np.float32(rng.uniform(0, 8, 5000))) + [np.float32(m) for m in _midpoints(grid)]
    for x in xs:
        x = float(x)
        want = _brute_encode(x, grid)
        assert oracle.e2m1_encode(x) == want, x
        assert oracle.e2m1_encode(-x) == want | 0x8, x


def test_e2m1_midpoints_round_to_even_code():
    # midpoint -> expected code (value): ties go to the code with an even index
    cases = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for x, c in cases.items():
        assert oracle.e2m1_encode(x) == c, x


def test_e2m1_saturation_and_signed_zero():
    assert oracle.e2m1_encode(6.5) == 7
    assert oracle.e2m1_encode(100.0) == 7
    assert oracle.e2m1_encode(-100.0) == 15
    assert oracle.e2m1_encode(0.0) == 0
    assert oracle.e2m1_encode(-0.0) == 8
    assert oracle.e2m1_encode(-0.1) == 8  # rounds to zero, keeps the sign


def test_roundtrip_every_finite_code():
    for c in range(16):
        assert oracle.e2m1_encode(oracle.e2m1_decode(c)) == c
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(10)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        np.float32(np.exp(rng.uniform(-80, 80, 5000)))])
    # exact ties: bf16 value + half an ulp
    ties = (rng.integers(0, 0x7F80, 1000, dtype=np.uint32) << 16) | 0x8000  # finite only
    x = np.concatenate([x, ties.view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16_bits(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, ref)


def _f16_table():
    """Every finite IEEE binary16 value (as float64) with its bit pattern, decoded from the format
    definition: sign, 5-bit exponent (bias 15), 10-bit mantissa; exponent 0 is subnormal."""
    bits = np.arange(0, 0x7c00, dtype=np.uint32)
    e = (bits >> 10) & 0x1f
    m = bits & 0x3ff
    val = np.where(e == 0, m * 2.0 ** -24, (1024 + m) * 2.0 ** (e.astype(np.int64) - 25))
    return val, bits


def test_f16_rounding_matches_torch_and_overflows_to_inf():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(50000) * np.exp2(rng.integers(-30, 18, 50000))).astype(np.float32)
    edge = np.array([65504, 65519.99, 65520, 65536, 1e30, -1e30, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                     2.0 ** -14 - 2.0 ** -25, 0.0, -0.0, np.inf, -np.inf], np.float32)
    x = np.concatenate([x, edge])
    got = oracle.round_out(x, "f16")
    want = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    assert oracle.f32_to_f16_bits(65520.0) == 0x7c00 and oracle.f32_to_f16_bits(-65520.0) == 0xfc00
    assert oracle.f32_to_f16_bits(65519.0) == 0x7bff


def test_f16_rounding_is_the_nearest_value_ties_to_even_by_brute_force():
    """Argmin over all finite f16 values (ties to the even mantissa) on random fp32 inputs and on
    every exact midpoint between neighbouring f16 values below 2^-10, plus a sample above."""
    val, bits = _f16_table()
    rng = np.random.default_rng(6)
    x = np.abs(rng.standard_normal(3000) * np.exp2(rng.integers(-26, 15, 3000))).astype(np.float32)
    mids = ((val[:-1] + val[1:]) / 2)
    x = np.concatenate([x, mids[val[1:] < 2.0 ** -10].astype(np.float32), mids[::97].astype(np.float32)])
    x = x[x.astype(np.float64) < 65504.0]  # finite results only; overflow is pinned above
    for v in x:
        d = np.abs(val - float(v))
        cand = np.flatnonzero(d == d.min())
        best = cand[0] if len(cand) == 1 else cand[(bits[cand] & 1) == 0][0]
        assert oracle.f32_to_f16_bits(float(v)) == bits[best], (float(v), hex(bits[best]))
        assert oracle.f32_to_f16_bits(-float(v)) == (bits[best] | 0x8000 if val[best] != 0 else 0x8000)


def test_splitk_reduce_f16_output_definition():
    """out = f16_rn(((p0 + p1) + p2) * g), the fp32 sum in split order: 2^24 + 1 - 2^24 in that
    order is 0, a product past 65520 is +inf, and a representable result is exact."""
    p = np.array([[[2.0 ** 24, 3.0, 1.0, 65000.0]], [[1.0, 5.0, 2.0, 500.0]],
                  [[-(2.0 ** 24), 0.5, 65503.0, 20.0]]], np.float32)
    got = oracle.splitk_reduce(p, np.float32(1.0), "f16")
    assert got[0, 0] == 0x0000  # (2^24 + 1) rounds to 2^24 in fp32, minus 2^24 = 0
    assert got[0, 1] == 0x4840  # 8.5 = 1.0625 * 2^3
    assert got[0, 2] == 0x7bff  # 65506 < 65520: rounds to 65504, the largest finite f16
    assert got[0, 3] == 0x7c00  # 65520 and above: +inf
    assert np.array_equal(oracle.splitk_reduce(p, np.float32(1.0)), oracle.splitk_reduce(p, np.float32(1.0), "bf16"))
