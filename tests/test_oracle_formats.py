"""Pins for the oracle's element formats (CPU only).

Each encoder is checked against an independent brute-force nearest search
written here with exact rational arithmetic, over every grid point, every
midpoint and the floats on either side of each midpoint; the decoders are
checked against hand-worked tables in tests/golden and against torch's own
float8_e4m3fn / bfloat16 conversions.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import formats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                rows.append((int(c, 0), float(v)))
    return rows


def _neighbours(v):
    v = np.float32(v)
    return [np.nextafter(v, np.float32(-np.inf)), v, np.nextafter(v, np.float32(np.inf))]


# ---------------------------------------------------------------- e2m1

def test_e2m1_table_matches_definition():
    for code, value in _read_table("e2m1_table.txt"):
        got = formats.e2m1_decode(code)
        assert got == value and np.signbit(got) == np.signbit(value), code


def _e2m1_brute(x):
    """Nearest e2m1 magnitude by exhaustive search; tie -> even code; saturating."""
    mags = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
            Fraction(3), Fraction(4), Fraction(6)]
    a = abs(Fraction(float(x)))
    if a >= 6:
        best = 7
    else:
        dists = [abs(a - m) for m in mags]
        d = min(dists)
        cands = [i for i, di in enumerate(dists) if di == d]
        best = [c for c in cands if c % 2 == 0][0] if len(cands) > 1 else cands[0]
    return best | (8 if np.signbit(np.float32(x)) else 0)


def test_e2m1_encode_brute_force():
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    pts = set()
    for g in grid:
        pts.update(_neighbours(g))
    for lo, hi in zip(grid[:-1], grid[1:]):
        pts.update(_neighbours((lo + hi) / 2))
    pts.update(_neighbours(7.0))
    pts.update([np.float32(100.0), np.float32(1e30), np.float32(1e-30), np.float32(0.0)])
    rng = np.random.default_rng(7)
    pts.update(rng.uniform(0, 8, 4000).astype(np.float32).tolist())
    xs = np.array(sorted(float(p) for p in pts), dtype=np.float32)
    xs = np.concatenate([xs, -xs])
    got = formats.e2m1_encode(xs)
    want = np.array([_e2m1_brute(x) for x in xs], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)


def test_e2m1_ties_go_to_even():
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for x, code in ties.items():
        assert formats.e2m1_encode(np.float32(x)) == code
        assert formats.e2m1_encode(np.float32(-x)) == code | 8


def test_e2m1_negative_zero_keeps_sign():
    assert formats.e2m1_encode(np.float32(-0.1)) == 8
    assert formats.e2m1_encode(np.float32(0.1)) == 0


# ---------------------------------------------------------------- ue4m3

def _ue4m3_values():
    return [Fraction(formats.ue4m3_decode(c).item()) for c in range(127)]


def _ue4m3_brute(x, vals):
    a = Fraction(float(x))
    if a >= 448:
        return 126
    dists = [abs(a - v) for v in vals]
    d = min(dists)
    cands = [i for i, di in enumerate(dists) if di == d]
    if len(cands) > 1:
        cands = [c for c in cands if c % 2 == 0]
    return cands[0]


def test_ue4m3_golden_points():
    for code, value in _read_table("ue4m3_points.txt"):
        assert formats.ue4m3_decode(code) == value
        assert formats.ue4m3_encode(np.float32(value)) == code


def test_ue4m3_decode_matches_torch():
    codes = torch.arange(0, 127, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(formats.ue4m3_decode(np.arange(127)), ref)


def test_ue4m3_encode_brute_force():
    vals = _ue4m3_values()
    pts = set()
    for v in vals:
        pts.update(_neighbours(float(v)))
    for lo, hi in zip(vals[:-1], vals[1:]):
        pts.update(_neighbours(float((lo + hi) / 2)))
    pts.update(_neighbours(464.0))
    pts.update(_neighbours(480.0))
    pts.update([np.float32(1e6), np.float32(2.0 ** -10), np.float32(2.0 ** -11), np.float32(0.0)])
    rng = np.random.default_rng(11)
    pts.update(np.exp2(rng.uniform(-12, 10, 3000)).astype(np.float32).tolist())
    xs = np.array(sorted(float(p) for p in pts if p >= 0), dtype=np.float32)
    got = formats.ue4m3_encode(xs)
    want = np.array([_ue4m3_brute(x, vals) for x in xs], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)


def test_ue4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(12)
    xs = np.exp2(rng.uniform(-12, np.log2(448.0), 20000)).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(formats.ue4m3_encode(xs), ref)


def test_ue4m3_saturates():
    assert formats.ue4m3_encode(np.float32(449.0)) == 0x7E
    assert formats.ue4m3_encode(np.float32(1e9)) == 0x7E


# ---------------------------------------------------------------- bf16

def test_bf16_round_matches_torch_for_float32_inputs():
    rng = np.random.default_rng(13)
    x = (rng.standard_normal(50000) * np.exp2(rng.integers(-40, 40, 50000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(formats.bf16_round(x.astype(np.float64)), ref)


def test_bf16_round_single_rounding_from_float64():
    # 1 + 2^-8 + 2^-30 lies just above the midpoint of two bf16 neighbours:
    # rounding straight from float64 goes up, while a detour through float32
    # (which drops the 2^-30) would land on the tie and go down to 1.0.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert formats.bf16_round(np.float64(x)) == 1.0 + 2.0 ** -7
    assert formats.bf16_round(np.float64(1.0 + 2.0 ** -8)) == 1.0          # tie -> even
    assert formats.bf16_round(np.float64(1.0 + 3 * 2.0 ** -8)) == 1.0 + 2 * 2.0 ** -7
    assert formats.bf16_round(np.float64(-3.0)) == -3.0


def test_bf16_bits_roundtrip():
    bits = np.arange(0, 65536, 7, dtype=np.uint32).astype(np.uint16)
    finite = np.isfinite(formats.bf16_bits_to_float(bits))
    b = bits[finite]
    np.testing.assert_array_equal(formats.float_to_bf16_bits(formats.bf16_bits_to_float(b)), b)
