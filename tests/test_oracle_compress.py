"""Pins of the oracle's sequence compressor (m tokens -> one FP4 entry).

[B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型", section
"CSA2：三层压缩一次吃满": every m tokens are compressed into one entry along the sequence.
The learned weights are not on the pages; the op takes the caller's per-token weights.
Each pin reduces the compressor to something fixed independently of its own loop: the FP4
quantiser on a single token, exact sums of small integers, and the E4M3 binade structure.
"""
import numpy as np
import pytest

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("ratio", [1, 2, 4, 8])
def test_one_hot_weights_select_one_token(ratio):
    """w[e] = unit vector k(e): the entry is token ratio*e + k(e), quantised alone."""
    rng = _rng(ratio)
    entries, dim = 37, 512
    x = rng.standard_normal((entries * ratio, dim)).astype(np.float32)
    k = rng.integers(0, ratio, entries)
    w = np.zeros((entries, ratio), np.float32)
    w[np.arange(entries), k] = 1.0
    codes, scales = oracle.compress_fp4(x, ratio, w)
    ref_c, ref_s = oracle.quantize_fp4(x[np.arange(entries) * ratio + k])
    assert np.array_equal(codes, ref_c) and np.array_equal(scales, ref_s)


def test_mean_of_equal_tokens_is_the_token():
    """w = None (the mean, 1/m): m copies of a short-mantissa row average to that row exactly."""
    rng = _rng(7)
    entries, dim, ratio = 20, 64, 4
    base = (rng.integers(-64, 64, (entries, dim)) / 8.0).astype(np.float32)   # 7-bit values
    x = np.repeat(base, ratio, axis=0)
    codes, scales = oracle.compress_fp4(x, ratio)
    ref_c, ref_s = oracle.quantize_fp4(base)
    assert np.array_equal(codes, ref_c) and np.array_equal(scales, ref_s)


def test_integer_sums_are_exact():
    """Small-integer tokens and weights 0/1/2: the weighted sum is exact in any order."""
    rng = _rng(11)
    entries, dim, ratio = 25, 128, 4
    x = rng.integers(-50, 50, (entries * ratio, dim)).astype(np.float32)
    w = rng.integers(0, 3, (entries, ratio)).astype(np.float32)
    codes, scales = oracle.compress_fp4(x, ratio, w)
    exact = (x.reshape(entries, ratio, dim).astype(np.float64) * w[:, :, None]).sum(axis=1)
    ref_c, ref_s = oracle.quantize_fp4(exact.astype(np.float32))
    assert np.array_equal(codes, ref_c) and np.array_equal(scales, ref_s)


def test_doubling_weights_moves_scales_one_binade():
    """Weights x2 double every entry: same E2M1 codes, E4M3 scale codes +8 (exponent + 1) while
    the scale stays a normal E4M3 number below 224."""
    rng = _rng(3)
    entries, dim, ratio = 30, 256, 4
    x = rng.standard_normal((entries * ratio, dim)).astype(np.float32)
    w = rng.uniform(0.1, 1.0, (entries, ratio)).astype(np.float32)
    c1, s1 = oracle.compress_fp4(x, ratio, w)
    c2, s2 = oracle.compress_fp4(x, ratio, 2 * w)
    normal = (s1 >= 8) & (s1 < 0x76)          # exponent field >= 1, value < 224
    assert normal.mean() > 0.9
    assert np.array_equal(s2[normal], s1[normal] + 8)
    blk = np.repeat(normal, 8, axis=1)         # 8 code bytes per 16-channel block
    assert np.array_equal(c2[blk], c1[blk])


def test_zero_weights_give_zero_entry():
    x = _rng(5).standard_normal((8, 64)).astype(np.float32)
    codes, scales = oracle.compress_fp4(x, 4, np.zeros((2, 4), np.float32))
    assert not codes.any() and not scales.any()
