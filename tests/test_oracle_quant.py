"""Pins for the oracle's quantise-on-write (FP4 main KV / indexer, FP8 sliding window).

The reference is exact-rational enumeration (tests/_exact.py): scale = nearest E4M3 to
amax/6, code = nearest E2M1 to x/scale; for the window, code = nearest E4M3 to x/s with
s = amax/448 rounded to fp32 (computed here by PyTorch).
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
from tests import _exact


def _fp4_blocks(rng, n):
    x = rng.standard_normal((n, 16)).astype(np.float32)
    x *= np.exp2(rng.integers(-14, 10, (n, 1))).astype(np.float32)
    x[0] = 0.0                                   # zero block -> zero scale, zero codes
    x[1] = 0.0
    x[1, 5] = -1e-4                              # tiny block: scale underflows to 0
    x[2, :] = np.float32(6.0) * np.arange(16, dtype=np.float32) / 15
    x[3, 3] = 1e5                                # saturating scale
    return x.reshape(-1, 64) if n % 4 == 0 else x


def test_fp4_quantize_matches_exact_enumeration():
    rng = np.random.default_rng(1)
    x = _fp4_blocks(rng, 160).reshape(-1, 64)
    codes, scales = oracle.quantize_fp4(x)
    for r in range(x.shape[0]):
        for b in range(4):
            blk = x[r, b * 16:(b + 1) * 16]
            amax = max(abs(Fraction(float(v))) for v in blk)
            sc = _exact.e4m3_encode(amax / 6, False)
            assert scales[r, b] == sc, (r, b)
            s = _exact.e4m3_value(sc)
            for i in range(16):
                c = b * 16 + i
                byte = codes[r, c // 2]
                got = (byte >> 4) if c & 1 else (byte & 15)
                exp = 0 if s == 0 else _exact.e2m1_encode(Fraction(float(blk[i])) / s, blk[i] < 0)
                assert got == exp, (r, c, float(blk[i]), float(s))


def test_fp4_nibble_order_and_zero_block():
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 1] = 6.0, 3.0          # amax 6 -> scale 1.0 (E4M3 0x38)
    codes, scales = oracle.quantize_fp4(x)
    assert scales[0, 0] == 0x38
    assert codes[0, 0] == 0x57           # element 0 -> low nibble (code 7), element 1 -> high (5)
    assert scales[0, 1] == 0 and not codes[0, 8:].any()


def test_fp4_roundtrip_error_bound():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    codes, scales = oracle.quantize_fp4(x)
    dq = oracle.dequantize_fp4(codes, scales)
    s = np.repeat(np.array([[oracle.e4m3_value(c) for c in row] for row in scales]), 16, axis=1)
    # inside the grid the error is at most half a grid step (<= 1 * s); the top element may
    # also lose what the rounded-down scale cannot reach (x/s <= 6 * 1.0625).
    assert np.all(np.abs(dq - x) <= 1.0 * s + 1e-12)
    assert np.all(np.abs(dq) <= 6 * s + 1e-12)


def test_fp8_token_matches_exact_enumeration():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((24, 512)).astype(np.float32)
    x[:, [7, 100]] *= 8
    x[5] = 0.0
    x[6] *= np.float32(1e-30)
    codes, scales = oracle.quantize_fp8_token(x)
    amax = torch.from_numpy(np.abs(x).max(axis=1))
    s_ref = (amax / torch.tensor(448.0, dtype=torch.float32)).numpy()
    assert np.array_equal(scales.view(np.uint32), s_ref.view(np.uint32))
    for r in range(x.shape[0]):
        s = Fraction(float(scales[r]))
        for i in range(0, 512, 7):
            exp = 0 if s == 0 else _exact.e4m3_encode(Fraction(float(x[r, i])) / s, x[r, i] < 0)
            assert codes[r, i] == exp, (r, i)
    assert not codes[5].any()


def test_fp8_token_vs_torch_conversion():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    codes, scales = oracle.quantize_fp8_token(x)
    q = torch.from_numpy(x).double() / torch.from_numpy(scales).double()[:, None]
    ref = q.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.mean(codes == ref) > 0.9999
