"""Pins for the oracle's number formats (E2M1 codes, E4M3 scales), independent of it.

Pins: the E2M1 grid and rounding cases (tests/golden), all 256 E4M3 codes against
PyTorch's float8_e4m3fn, and nearest-value enumeration in exact rationals.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_pairs(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            rows.append((a, b))
    return rows


def test_e2m1_grid_matches_golden():
    for code, val in _read_pairs("e2m1_grid.txt"):
        v = oracle.e2m1_value(int(code))
        assert v == float(val)
        assert math.copysign(1.0, v) == math.copysign(1.0, float(val))


def test_e2m1_rounding_matches_golden():
    for val, code in _read_pairs("e2m1_rounding.txt"):
        assert oracle.e2m1_encode(float(val)) == int(code), val


def _e4m3_table():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_all_codes_vs_torch():
    table = _e4m3_table()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if math.isnan(table[c]):
            assert math.isnan(v), c
        else:
            assert v == table[c], c
            assert math.copysign(1, v) == math.copysign(1, table[c]), c


def _nearest_e4m3_exact(x: Fraction) -> int:
    """Independent encoder: enumerate the finite E4M3 magnitudes, nearest with ties to the
    even code, saturate at 448, keep the sign."""
    table = _e4m3_table()
    sign = 0x80 if x < 0 or (x == 0 and False) else 0
    a = abs(x)
    best, best_err = None, None
    for c in range(0x7F):            # finite non-negative codes 0..0x7E
        err = abs(Fraction(table[c]) - a)
        if best is None or err < best_err or (err == best_err and c % 2 == 0):
            best, best_err = c, err
    return sign | best


def test_e4m3_encode_vs_enumeration():
    rng = np.random.default_rng(123)
    vals = list(rng.standard_normal(300) * np.exp2(rng.integers(-12, 9, 300)))
    table = _e4m3_table()
    # every midpoint between neighbouring finite magnitudes, and the codes themselves
    for c in range(0x7E):
        vals.append((table[c] + table[c + 1]) / 2)
        vals.append(table[c])
    vals += [448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -12]
    for v in vals:
        got = oracle.e4m3_encode(float(v))
        exp = _nearest_e4m3_exact(Fraction(float(v)))
        if v < 0:
            exp |= 0x80
        assert got == exp, (v, got, exp)


def test_e4m3_encode_vs_torch_in_range():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-14, 8, 20000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_satfinite():
    # torch turns these into NaN; the quantiser saturates (reading: satfinite).
    for v in [449.0, 464.0, 500.0, 1e9]:
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE


def test_negative_underflow_keeps_sign():
    assert oracle.e4m3_encode(-1e-6) == 0x80
    assert oracle.e2m1_encode(-1e-6) == 0x8
