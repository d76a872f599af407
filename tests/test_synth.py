"""The seeded generator is deterministic and per-sequence streams are independent."""
import numpy as np

from compressed_sparse_attention_quantize_b200 import synth


def test_deterministic_and_shapes():
    wl = synth.workload(0)
    a = synth.kv_latent(wl, 0)
    b = synth.kv_latent(wl, 0)
    assert a.shape == (1024, 512) and a.dtype == np.float32 and np.array_equal(a, b)
    oc = synth.outlier_channels(wl.seed)
    assert len(set(oc.tolist())) == 4
    assert np.abs(a[:, oc]).mean() > 5 * np.abs(np.delete(a, oc, axis=1)).mean()
    assert synth.main_query_bf16(wl, 0, 0).shape == (1, 16, 512)
    assert synth.index_query(wl, 0, 0).shape == (1, 4, 64)
    w = synth.head_weights(wl, 0, 0)
    assert w.shape == (1, 4) and (w >= 0).all() and (w < 1).all()


def test_workloads():
    w3 = synth.workload(3)
    assert w3.B == 4 and all(131072 <= n <= 262144 for n in w3.n_entries)
    w4 = synth.workload(4)
    qp = w4.q_pos(0)
    assert qp[0] == 4 * 32768 and qp[-1] == 4 * 32768 + 4095
    st, ln = synth.swa_window(w4, 0)
    assert st[0] == 0 and ln[0] == 128 and st[-1] == 4095
    w1 = synth.workload(1)
    st, ln = synth.swa_window(w1, 0)
    assert ln[0] == 128 and w1.modes == ("F", "U", "U", "U", "U", "U")


def test_window_extents_follow_the_reading():
    """Window slots [start, start + len) of query t hold tokens max(0, p - 127) .. p (prefill:
    slot s holds token prefill_start - 127 + s); decode sees the whole filled ring."""
    wl = synth.scaled(synth.workload(4), n=2000, T=96, K=256, name="prefill_scaled")
    first = wl.prefill_start - (synth.SWA_WINDOW - 1)
    st, ln = synth.swa_window(wl, 0)
    for t, p in enumerate(wl.q_pos(0)):
        tokens = first + np.arange(st[t], st[t] + ln[t])
        assert tokens[0] == max(0, int(p) - 127) and tokens[-1] == p and ln[t] == min(128, int(p) + 1)
        assert st[t] + ln[t] <= wl.swa_tokens()
    w1 = synth.workload(1)
    st, ln = synth.swa_window(w1, 3)
    assert st[0] == 0 and ln[0] == 128
