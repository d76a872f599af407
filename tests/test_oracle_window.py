"""Pins of the oracle's sliding-window reading (the last 128 tokens up to the query).

The oracle lists, from the definition, the tokens u with p - 128 < u <= p and u >= 0.  These
tests check it against the closed form (a contiguous run of min(128, p + 1) tokens ending at p),
against brute-force membership, against the window size parameter, and on the workloads' own
queries; and they check that the window buffers the workloads lay out hold exactly those tokens.
"""
import numpy as np

import oracle
from compressed_sparse_attention_quantize_b200 import synth


def test_closed_form():
    assert oracle.window_tokens(-1).size == 0
    for p in list(range(0, 300)) + [131071, 1 << 20]:
        w = oracle.window_tokens(p)
        n = min(128, p + 1)
        assert w.size == n, p
        assert w[-1] == p and w[0] == max(0, p - 127), p
        assert np.array_equal(w, np.arange(p - n + 1, p + 1)), p


def test_brute_force_membership_and_size_parameter():
    for p in (0, 5, 127, 128, 200):
        for W in (1, 4, 128):
            w = set(oracle.window_tokens(p, W).tolist())
            for u in range(0, p + 1):
                assert (u in w) == (p - u < W), (p, W, u)


def _slots_of(wl, b, t):
    qp = int(wl.q_pos(b)[t])
    return [synth.window_slot(wl, b, u) for u in oracle.window_tokens(qp)]


def test_workload_buffers_hold_the_window():
    """The slot range a query reads (synth.swa_window) holds exactly the oracle's window tokens."""
    cases = [synth.workload(1), synth.workload(3),
             synth.scaled(synth.workload(1), B=3, n=[0, 20, 37], name="short"),
             synth.scaled(synth.workload(4), n=2000, T=96, K=256, name="prefill_scaled")]
    for wl in cases:
        for b in range(wl.B):
            st, ln = synth.swa_window(wl, b)
            for t in sorted({0, min(1, wl.T - 1), wl.T // 2, wl.T - 1}):
                slots = _slots_of(wl, b, t)
                assert sorted(slots) == list(range(int(st[t]), int(st[t]) + int(ln[t]))), (wl.name, b, t)
                assert all(0 <= s < wl.swa_tokens() for s in slots)
