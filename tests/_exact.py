"""Independent exact-rational encoders used to pin the oracle (tests only).

They enumerate the representable values (E2M1 grid from tests/golden, E4M3 values from
PyTorch's float8_e4m3fn) and pick the nearest in exact rationals, ties to the even code.
"""
import os
from fractions import Fraction
from functools import lru_cache

import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@lru_cache(None)
def e2m1_grid():
    vals = []
    with open(os.path.join(GOLDEN, "e2m1_grid.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                vals.append(Fraction(float(v)))
    return vals[:8]          # non-negative magnitudes, codes 0..7


@lru_cache(None)
def e4m3_mags():
    codes = torch.arange(0x7F, dtype=torch.int32).to(torch.uint8)
    return [Fraction(float(v)) for v in codes.view(torch.float8_e4m3fn).to(torch.float64)]


def _nearest(table, a):
    best, best_err = 0, None
    for c, v in enumerate(table):
        err = abs(v - a)
        if best_err is None or err < best_err or (err == best_err and c % 2 == 0):
            best, best_err = c, err
    return best


def e2m1_encode(x: Fraction, negative: bool) -> int:
    return (8 if negative else 0) | _nearest(e2m1_grid(), abs(x))


def e4m3_encode(x: Fraction, negative: bool) -> int:
    return (0x80 if negative else 0) | _nearest(e4m3_mags(), abs(x))


def e4m3_value(code: int) -> Fraction:
    v = e4m3_mags()[code & 0x7F]
    return -v if code & 0x80 else v


def e2m1_value(code: int) -> Fraction:
    v = e2m1_grid()[code & 7]
    return -v if code & 8 else v
