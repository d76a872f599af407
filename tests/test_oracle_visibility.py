"""Pins of the oracle's causal visibility rule (prefill).

The oracle counts, from the definition, the entries j with 4j + 3 <= p.  These tests check it
against the closed form min(n, floor((p + 1) / 4)), against the step structure (one more entry
exactly when p completes a group of four tokens), and on the prefill workload's first and last
query.
"""
import oracle
from compressed_sparse_attention_quantize_b200 import synth


def test_closed_form_and_steps():
    for n in (0, 1, 7, 100):
        prev = oracle.visible_entries(-1, n)
        assert prev == 0
        for p in range(0, 420):
            v = oracle.visible_entries(p, n)
            assert v == min(n, (p + 1) // 4), (n, p)
            assert v - prev == (1 if (p % 4 == 3 and prev < n) else 0), (n, p)
            prev = v


def test_decode_sees_every_entry():
    assert oracle.visible_entries(None, 0) == 0
    assert oracle.visible_entries(None, 32768) == 32768


def test_prefill_workload_ends():
    wl = synth.workload(4)
    qp = wl.q_pos(0)
    n = wl.n_entries[0]
    assert oracle.visible_entries(int(qp[0]), n) == 32768        # the chunk's first token
    assert oracle.visible_entries(int(qp[-1]), n) == 33792       # all 1024 new entries complete


def test_bench_accounting_matches_the_oracle():
    """bench.py counts algorithmic bytes with its own copy of the rule; it must agree."""
    import bench
    for i in range(5):
        wl = synth.workload(i)
        for b in range(wl.B):
            got = bench.visible_counts(wl, b)
            if wl.prefill_start is None:
                assert got.tolist() == [oracle.visible_entries(None, wl.n_entries[b])]
            else:
                qp = wl.q_pos(b)
                for t in (0, 1, 2, 3, len(qp) // 2, len(qp) - 1):
                    assert int(got[t]) == oracle.visible_entries(int(qp[t]), wl.n_entries[b])
