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
