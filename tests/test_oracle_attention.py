"""Pins for the oracle's attention over selected entries + the 8-bit window.

Pins: single-entry and equal-logit closed forms, dense attention (top-K >= n) against an
independent numpy softmax, exact high-precision brute force (mpmath) on a tiny case,
LSE against scipy, empty input, and the Reuse identity.
"""
import mpmath
import numpy as np
from scipy.special import logsumexp

import oracle
from compressed_sparse_attention_quantize_b200 import synth


def _bf16_bits(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((u + ((u >> 16) & 1) + np.uint32(0x7FFF)) >> 16).astype(np.uint16)


def _bf16_value(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _case(rng, H, n, nswa):
    kv = rng.standard_normal((n, 512)).astype(np.float32)
    kv[:, [3, 77]] *= 8
    kc, ks = oracle.quantize_fp4(kv)
    rows = oracle.pack_kv_rows(kc, ks)
    sw = rng.standard_normal((nswa, 512)).astype(np.float32)
    swc, sws = oracle.quantize_fp8_token(sw) if nswa else (np.zeros((0, 512), np.uint8),
                                                           np.zeros(0, np.float32))
    q = _bf16_bits(rng.standard_normal((H, 512)) / np.sqrt(512))
    return rows, kc, ks, swc, sws, q


def _values(kc, ks, swc, sws, idx):
    v = oracle.dequantize_fp4(kc, ks)[[i for i in idx if i >= 0]]
    if len(swc):
        e4 = np.array([oracle.e4m3_value(c) for c in range(256)])
        v = np.concatenate([v, e4[swc] * sws.astype(np.float64)[:, None]])
    return v


def test_single_entry_returns_its_value():
    rng = np.random.default_rng(20)
    rows, kc, ks, swc, sws, q = _case(rng, 4, 10, 0)
    idx = np.array([7, -1, -1], np.int32)
    out, lse = oracle.attention(q, rows, idx, swc, sws, 1.0)
    v = oracle.dequantize_fp4(kc, ks)[7]
    assert np.array_equal(out, np.tile(v, (4, 1)))
    z = (_bf16_value(q) @ v)
    assert np.allclose(lse, z, rtol=1e-14, atol=1e-14)


def test_equal_logits_give_plain_mean():
    rng = np.random.default_rng(21)
    rows, kc, ks, swc, sws, _ = _case(rng, 2, 50, 9)
    q = np.zeros((2, 512), np.uint16)
    idx = np.array([1, 4, 9, 33, -1], np.int32)
    out, lse = oracle.attention(q, rows, idx, swc, sws, 0.5)
    v = _values(kc, ks, swc, sws, idx)
    assert np.allclose(out, v.mean(axis=0)[None], rtol=1e-13, atol=1e-13)
    assert np.allclose(lse, np.log(len(v)))


def test_dense_when_k_covers_all_entries():
    rng = np.random.default_rng(22)
    H, n = 8, 300
    rows, kc, ks, swc, sws, q = _case(rng, H, n, 128)
    idx = np.arange(n, dtype=np.int32)
    for scale in (1.0, 1 / np.sqrt(512)):
        out, lse = oracle.attention(q, rows, idx, swc, sws, scale)
        V = _values(kc, ks, swc, sws, idx)
        z = scale * (_bf16_value(q) @ V.T)
        p = np.exp(z - z.max(axis=1, keepdims=True))
        ref = (p @ V) / p.sum(axis=1, keepdims=True)
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, logsumexp(z, axis=1), rtol=1e-13)


def test_mpmath_brute_force_tiny():
    rng = np.random.default_rng(23)
    rows, kc, ks, swc, sws, q = _case(rng, 2, 6, 3)
    idx = np.array([5, 0, 2], np.int32)
    out, lse = oracle.attention(q, rows, idx, swc, sws, 1.0)
    mpmath.mp.dps = 40
    V = _values(kc, ks, swc, sws, idx)
    qv = _bf16_value(q)
    for h in range(2):
        z = [mpmath.fsum(mpmath.mpf(float(a)) * mpmath.mpf(float(b)) for a, b in zip(qv[h], V[x]))
             for x in range(len(V))]
        e = [mpmath.exp(zz) for zz in z]
        l = mpmath.fsum(e)
        for d in range(0, 512, 37):
            ref = mpmath.fsum(e[x] * mpmath.mpf(float(V[x, d])) for x in range(len(V))) / l
            assert abs(out[h, d] - float(ref)) <= 1e-12 * (1 + abs(float(ref)))
        assert abs(lse[h] - float(mpmath.log(l))) <= 1e-12


def test_empty_row():
    rows = np.zeros((1, 288), np.uint8)
    q = np.zeros((2, 512), np.uint16)
    out, lse = oracle.attention(q, rows, np.full(4, -1, np.int32), np.zeros((0, 512), np.uint8),
                                np.zeros(0, np.float32), 1.0)
    assert not out.any() and np.all(np.isneginf(lse))


def test_reuse_identity_and_synth_shapes():
    wl = synth.scaled(synth.workload(1), B=1, n=256, K=16)
    k = synth.index_keys(wl, 0)
    kc, ks = oracle.quantize_fp4(k)
    rows = oracle.pack_kv_rows(*oracle.quantize_fp4(synth.kv_latent(wl, 0)))
    iq = synth.index_query(wl, 0, 0)[0]
    qc, qs = oracle.quantize_fp4(iq)
    w = synth.head_weights(wl, 0, 0)[0]
    idx, cnt, _, _, _ = oracle.full_index(qc, qs, w, kc, ks, 256, 16)
    swc, sws = oracle.quantize_fp8_token(synth.swa_latent(wl, 0, 0))
    q = synth.main_query_bf16(wl, 0, 0)[0]
    full = oracle.attention(q, rows, idx, swc, sws, 1 / np.sqrt(512))
    group = oracle.layer_group_indices(("F", "U"), [(qc, qs, w), None], kc, ks, 256, 16, 0)
    reuse = oracle.attention(q, rows, group[1][0], swc, sws, 1 / np.sqrt(512))
    assert np.array_equal(full[0], reuse[0]) and np.array_equal(full[1], reuse[1])
    assert q.shape == (64, 512) and rows.shape == (256, 288) and swc.shape == (128, 512)
