"""Pins of the oracle's pool maintenance across decode steps.

The rule: every R steps the Full layer's scan rebuilds the pool (top-min(P, n) of its order) and
records the entry count n_ref; in between, Reindex layers search the kept pool followed by the
entries written since (n_ref .. n - 1).  Pins: R = 1 is the per-step rebuild step by step; the
extension's closed form; the Full layer's own selection does not depend on R; every Reindex
selection between refreshes equals an independent float64 score + numpy lexsort over exactly
the kept pool and the new entries; with a pool that holds the whole context the kept pool plus
the new entries is the whole context again.
"""
import numpy as np

import oracle

MODES = ("F", "I", "U", "I")


def _quant_rows(x):
    return oracle.quantize_fp4(np.ascontiguousarray(x, np.float32))


def _setup(seed, n_max, steps, H=4):
    rng = np.random.default_rng(seed)
    kc, ks = _quant_rows(rng.standard_normal((n_max, 64)))
    inputs = []
    for s in range(steps):
        per = []
        for m in MODES:
            if m == "U":
                per.append(None)
                continue
            qc, qs = _quant_rows(rng.standard_normal((H, 64)) / 8)
            per.append((qc, qs, rng.random(H).astype(np.float32)))
        inputs.append(per)
    return kc, ks, inputs


def _dequant(codes, scales):
    return oracle.dequantize_fp4(codes, scales)


def _lexsort_topk(qc, qs, w, kc, ks, cand, K):
    """Independent selection: the score in the stated fixed fp32 order from exactly dequantised
    values (float64 block partials are exact), ranked by numpy lexsort."""
    q = _dequant(qc, qs)
    k = _dequant(kc[cand], ks[cand])
    sc = np.zeros(len(cand), np.float32)
    for h in range(q.shape[0]):
        blocks = [(k[:, 16 * b:16 * b + 16] @ q[h, 16 * b:16 * b + 16]).astype(np.float32) for b in range(4)]
        dot = ((blocks[0] + blocks[1]) + blocks[2]) + blocks[3]
        sc = (sc + np.float32(w[h]) * np.maximum(dot, np.float32(0))).astype(np.float32)
    order = np.lexsort((np.asarray(cand), -sc.astype(np.float64)))[:K]
    chosen = np.sort(np.asarray(cand)[order]).astype(np.int32)
    out = np.full(K, -1, np.int32)
    out[:len(chosen)] = chosen
    return out


def test_extend_pool_closed_form():
    pool = np.array([3, 9, 40, 41, 77, -1, -1], np.int32)
    got = oracle.extend_pool(pool, 5, 80, 84)
    assert got.tolist() == [3, 9, 40, 41, 77, 80, 81, 82, 83]
    assert oracle.extend_pool(pool, 5, 80, 80).tolist() == [3, 9, 40, 41, 77]
    assert oracle.extend_pool(pool, 0, 5, 7).tolist() == [5, 6]


def test_refresh_every_step_is_the_per_step_rebuild():
    n_steps = [300, 301, 305, 305, 320]
    kc, ks, inputs = _setup(1, 320, len(n_steps))
    got = oracle.decode_steps_with_pool(MODES, inputs, kc, ks, n_steps, K=24, P=90, R=1)
    for s, n in enumerate(n_steps):
        ref = oracle.layer_group_indices(MODES, inputs[s], kc, ks, n, 24, 90)
        for (a, ca), (b, cb) in zip(got[s], ref):
            assert np.array_equal(a, b) and ca == cb


def test_between_refreshes_reindex_searches_kept_pool_and_new_entries():
    n_steps = [300, 302, 305, 306, 320, 321, 330]
    K, P, R = 24, 90, 3
    kc, ks, inputs = _setup(2, 330, len(n_steps))
    got = oracle.decode_steps_with_pool(MODES, inputs, kc, ks, n_steps, K=K, P=P, R=R)
    full_every = oracle.decode_steps_with_pool(MODES, inputs, kc, ks, n_steps, K=K, P=P, R=1)
    for s, n in enumerate(n_steps):
        # the Full layer's own selection is over the whole visible context whatever R is
        assert np.array_equal(got[s][0][0], full_every[s][0][0])
        base = s - s % R
        qc, qs, w = inputs[base][0]
        _, _, pool, pool_len, _ = oracle.full_index(qc, qs, w, kc, ks, n_steps[base], K, P)
        cand = np.concatenate([pool[:pool_len], np.arange(n_steps[base], n)]).astype(np.int32)
        for l, m in enumerate(MODES):
            if m == "I":
                qc, qs, w = inputs[s][l]
                assert np.array_equal(got[s][l][0], _lexsort_topk(qc, qs, w, kc, ks, cand, K)), (s, l)
            if m == "U":
                assert np.array_equal(got[s][l][0], got[s][l - 1][0])


def test_pool_of_the_whole_context_stays_whole():
    n_steps = [100, 103, 110]
    kc, ks, inputs = _setup(3, 110, len(n_steps))
    got = oracle.decode_steps_with_pool(MODES, inputs, kc, ks, n_steps, K=16, P=500, R=10)
    for s, n in enumerate(n_steps):
        for l, m in enumerate(MODES):
            if m == "I":
                qc, qs, w = inputs[s][l]
                ref, _ = oracle.reindex(qc, qs, w, kc, ks, np.arange(n, dtype=np.int32), n, 16)
                assert np.array_equal(got[s][l][0], ref)
