"""Pins for the oracle's indexer score, top-K, pool and layer modes.

Pins: exact-rational per-block dot products; an independent float64 numpy score; scale
and permutation invariants; exhaustive subset enumeration for top-K on tiny inputs;
numpy lexsort on larger ones; Reindex == Full when the pool is the whole context.
"""
import itertools
from fractions import Fraction

import numpy as np

import oracle
from tests import _exact


def _quant_rows(x):
    return oracle.quantize_fp4(np.ascontiguousarray(x, np.float32))


def _dequant_exact(codes, scales, r):
    vals = []
    for c in range(codes.shape[1] * 2):
        byte = codes[r, c // 2]
        code = (byte >> 4) if c & 1 else (byte & 15)
        vals.append(_exact.e2m1_value(code) * _exact.e4m3_value(scales[r, c // 16]))
    return vals


def _make(rng, H, n):
    q = (rng.standard_normal((H, 64)) / 8).astype(np.float32)
    k = rng.standard_normal((n, 64)).astype(np.float32)
    w = rng.random(H).astype(np.float32)
    qc, qs = _quant_rows(q)
    kc, ks = _quant_rows(k)
    return qc, qs, w, kc, ks


def test_score_blocks_exact_and_fixed_order():
    rng = np.random.default_rng(10)
    H, n = 4, 40
    qc, qs, w, kc, ks = _make(rng, H, n)
    s = oracle.index_scores(qc, qs, w, kc, ks)
    qv = [_dequant_exact(qc, qs, h) for h in range(H)]
    for j in range(n):
        kv = _dequant_exact(kc, ks, j)
        acc = np.float32(0)
        for h in range(H):
            p = [sum(qv[h][b * 16 + i] * kv[b * 16 + i] for i in range(16)) for b in range(4)]
            pf = [np.float32(float(x)) for x in p]
            assert all(Fraction(float(a)) == b for a, b in zip(pf, p))   # partials exact in fp32
            dot = np.float32(np.float32(np.float32(pf[0] + pf[1]) + pf[2]) + pf[3])
            acc = np.float32(acc + np.float32(w[h] * max(dot, np.float32(0))))
        assert s[j] == acc, j


def test_score_vs_float64_numpy():
    rng = np.random.default_rng(11)
    H, n = 8, 3000
    qc, qs, w, kc, ks = _make(rng, H, n)
    s = oracle.index_scores(qc, qs, w, kc, ks)
    q = oracle.dequantize_fp4(qc, qs)
    k = oracle.dequantize_fp4(kc, ks)
    ref = np.maximum(k @ q.T, 0) @ w.astype(np.float64)
    assert np.allclose(s, ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_score_invariants():
    rng = np.random.default_rng(12)
    qc, qs, w, kc, ks = _make(rng, 8, 500)
    s = oracle.index_scores(qc, qs, w, kc, ks)
    s2 = oracle.index_scores(qc, qs, w * np.float32(2), kc, ks)
    assert np.array_equal(s2, s * np.float32(2))             # power-of-two weight scale: exact
    perm = rng.permutation(500)
    sp = oracle.index_scores(qc, qs, w, kc[perm], ks[perm])
    assert np.array_equal(sp, s[perm])
    # negating the query flips every dot: only keys with all dots <= 0 score 0 both ways
    qneg = qc ^ np.uint8(0x88)
    sn = oracle.index_scores(qneg, qs, w, kc, ks)
    assert np.all(sn >= 0) and np.all(s >= 0)
    assert not np.any(np.signbit(s)) and not np.any(np.signbit(sn))


def _topk_by_enumeration(scores, K):
    n = len(scores)
    k = min(K, n)
    winners = []
    for S in itertools.combinations(range(n), k):
        Sset = set(S)
        ok = all((scores[i] > scores[j]) or (scores[i] == scores[j] and i < j)
                 for i in S for j in range(n) if j not in Sset)
        if ok:
            winners.append(S)
    assert len(winners) == 1
    return list(winners[0])


def test_topk_exhaustive_tiny_with_ties():
    rng = np.random.default_rng(13)
    for trial in range(60):
        n = int(rng.integers(0, 11))
        scores = rng.choice(np.array([0.0, 0.5, 1.0, 2.0, 3.5], np.float32), size=n)
        for K in range(0, n + 3):
            idx, cnt = oracle.topk(scores, K)
            exp = _topk_by_enumeration(list(scores), K)
            assert cnt == len(exp)
            assert list(idx[:cnt]) == sorted(exp)
            assert np.all(idx[cnt:] == -1)


def test_topk_vs_lexsort():
    rng = np.random.default_rng(14)
    s = np.round(rng.random(20000) * 300).astype(np.float32)     # many ties
    for K in (1, 64, 2048, 19999, 20000, 30000):
        idx, cnt = oracle.topk(s, K)
        order = np.lexsort((np.arange(len(s)), -s.astype(np.float64)))
        exp = np.sort(order[:min(K, len(s))])
        assert cnt == len(exp) and np.array_equal(idx[:cnt], exp)


def test_pool_nests_topk_and_reindex_identity():
    rng = np.random.default_rng(15)
    qc, qs, w, kc, ks = _make(rng, 8, 4000)
    idx, cnt, pool, plen, s = oracle.full_index(qc, qs, w, kc, ks, 4000, K=64, P=1000)
    assert cnt == 64 and plen == 1000
    assert set(idx[:cnt]) <= set(pool[:plen])
    # whole context as pool + same query -> Reindex picks the Full layer's top-K
    whole = np.arange(4000, dtype=np.int32)
    ri, rc = oracle.reindex(qc, qs, w, kc, ks, whole, 4000, K=64)
    assert rc == cnt and np.array_equal(ri, idx)
    # a positive power-of-two weight scale leaves the selection unchanged
    idx2, _, _, _, _ = oracle.full_index(qc, qs, w * np.float32(4), kc, ks, 4000, K=64)
    assert np.array_equal(idx2, idx)


def test_selection_independent_of_entry_order():
    rng = np.random.default_rng(16)
    qc, qs, w, kc, ks = _make(rng, 8, 3000)
    idx, cnt, _, _, s = oracle.full_index(qc, qs, w, kc, ks, 3000, K=100)
    perm = rng.permutation(3000)
    idxp, cntp, _, _, _ = oracle.full_index(qc, qs, w, kc[perm], ks[perm], 3000, K=100)
    sel = set(idx[:cnt].tolist())
    selp = set(perm[idxp[:cntp]].tolist())
    # the selected score multiset is label-free; entries strictly above the K-th score are
    # selected under any labelling (ties at the K-th score may resolve to other labels)
    assert sorted(s[list(sel)]) == sorted(s[list(selp)])
    t = np.sort(s)[::-1][99]
    above = set(np.nonzero(s > t)[0].tolist())
    assert above <= sel and above <= selp


def test_layer_group_modes():
    rng = np.random.default_rng(17)
    n = 2000
    k = rng.standard_normal((n, 64)).astype(np.float32)
    kc, ks = _quant_rows(k)
    inputs = []
    for _ in range(6):
        q = (rng.standard_normal((8, 64)) / 8).astype(np.float32)
        qc, qs = _quant_rows(q)
        inputs.append((qc, qs, rng.random(8).astype(np.float32)))
    modes = ("F", "I", "U", "I", "U", "U")
    res = oracle.layer_group_indices(modes, inputs, kc, ks, n, K=32, P=300)
    # Reuse copies the preceding layer
    assert np.array_equal(res[2][0], res[1][0]) and np.array_equal(res[4][0], res[3][0])
    assert np.array_equal(res[5][0], res[3][0])
    # Reindex picks from the Full layer's pool
    _, _, pool, plen, _ = oracle.full_index(*inputs[0], kc, ks, n, K=32, P=300)
    assert set(res[1][0]) <= set(pool[:plen]) and set(res[3][0]) <= set(pool[:plen])
    try:
        oracle.layer_group_indices(("U", "F"), inputs, kc, ks, n, 32, 300)
        raise AssertionError("Reuse before Full must be rejected")
    except ValueError:
        pass
