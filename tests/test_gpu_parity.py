"""CUDA path vs oracle, through the C ABI, on seeded synthetic inputs.

Bit-exact: FP4 codes and scales, FP8 window codes and scales, top-K index sets and pools.
Attention: relative L2 <= 1e-3 and max-abs <= 2e-3 * RMS(reference) per query row.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import compressed_sparse_attention_quantize_b200 as csa2
from compressed_sparse_attention_quantize_b200 import runtime, synth
from tests._parity import OracleSeq, check_attention

pytestmark = pytest.mark.gpu


def _special_rows(rng, rows, dim):
    x = rng.standard_normal((rows, dim)).astype(np.float32)
    x *= np.exp2(rng.integers(-20, 12, (rows, 1))).astype(np.float32)
    x[0] = 0.0
    x[1, :16] = np.float32(-1e-7)
    x[2, :16] = np.array([6, 5, 3.5, 2.5, 1.75, 1.25, .75, .25, -6, -5, -3.5, -2.5, -1.75, -1.25, -.75, -.25],
                         np.float32)
    x[3, 7] = 3e5
    x[4] = 448.0 * np.sin(np.arange(dim, dtype=np.float32))
    x[5, ::3] *= 8
    return x


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_fp4_bitexact(dtype):
    rng = np.random.default_rng(100)
    x = _special_rows(rng, 777, 512)
    xt = torch.from_numpy(x).cuda()
    if dtype == "bf16":
        xt = xt.to(torch.bfloat16)
        x = xt.float().cpu().numpy()
    codes = torch.zeros((777, 288), dtype=torch.uint8, device="cuda")
    runtime.quantize_fp4_rows(xt, codes, codes[:, 256:], 288, 288)
    torch.cuda.synchronize()
    oc, os_ = oracle.quantize_fp4(x)
    got = codes.cpu().numpy()
    assert np.array_equal(got[:, :256], oc)
    assert np.array_equal(got[:, 256:], os_)


def test_quantize_fp4_scatter_rows():
    rng = np.random.default_rng(101)
    x = rng.standard_normal((10, 64)).astype(np.float32)
    dst = torch.tensor([9, 3, 0, 17, 4, 5, 6, 7, 8, 1], dtype=torch.int64, device="cuda")
    codes = torch.zeros((20, 32), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((20, 4), dtype=torch.uint8, device="cuda")
    runtime.quantize_fp4_rows(torch.from_numpy(x).cuda(), codes, scales, 32, 4, dst_rows=dst)
    torch.cuda.synchronize()
    oc, os_ = oracle.quantize_fp4(x)
    d = dst.cpu().numpy()
    assert np.array_equal(codes.cpu().numpy()[d], oc)
    assert np.array_equal(scales.cpu().numpy()[d], os_)
    assert not codes.cpu().numpy()[[2, 10, 19]].any()


@pytest.mark.parametrize("dtype,ratio,weighted", [("f32", 4, True), ("bf16", 4, True), ("f32", 4, False),
                                                    ("f32", 3, True), ("bf16", 1, False), ("f32", 16, True)])
def test_compress_fp4_bitexact(dtype, ratio, weighted):
    """Compressor + quantise-on-write vs the oracle: packed 288-byte rows written at scattered
    destinations; padded token rows and a padded weight matrix."""
    rng = np.random.default_rng(200 + ratio)
    entries, dim = 523, 512
    x = rng.standard_normal((entries * ratio, dim)).astype(np.float32)
    x[:, rng.choice(dim, 4, replace=False)] *= 8.0                  # outlier channels
    x[::7] *= np.float32(1e-3)
    xpad = np.zeros((entries * ratio, dim + 32), np.float32)
    xpad[:, :dim] = x
    xt = torch.from_numpy(xpad).cuda()
    if dtype == "bf16":
        xt = xt.to(torch.bfloat16)
        x = xt[:, :dim].float().cpu().numpy()
    w = None
    wt = None
    if weighted:
        w = rng.uniform(-0.5, 1.0, (entries, ratio)).astype(np.float32)
        wpad = np.zeros((entries, ratio + 3), np.float32)
        wpad[:, :ratio] = w
        wt = torch.from_numpy(wpad).cuda()
    dst = torch.from_numpy(rng.permutation(entries + 40)[:entries].astype(np.int64)).cuda()
    rows = torch.zeros((entries + 40, 288), dtype=torch.uint8, device="cuda")
    csa2.csa2_compress_quantize_kv(xt, csa2.DTYPE_BF16 if dtype == "bf16" else csa2.DTYPE_F32, entries,
                                   ratio, dim, xt.stride(0), wt, ratio + 3, rows, 288, rows[:, 256:], 288,
                                   dst_rows=dst)
    torch.cuda.synchronize()
    oc, os_ = oracle.compress_fp4(x, ratio, w)
    got = rows.cpu().numpy()[dst.cpu().numpy()]
    assert np.array_equal(got[:, :256], oc)
    assert np.array_equal(got[:, 256:], os_)


def test_quantize_fp8_token_bitexact():
    rng = np.random.default_rng(102)
    x = _special_rows(rng, 300, 512)
    # rows whose scale is exactly 1 put many values on E4M3 ties
    x[10] = np.float32(448.0)
    x[10, 1:100] = np.linspace(200, 250, 99, dtype=np.float32)
    xt = torch.from_numpy(x).cuda()
    codes = torch.empty((300, 512), dtype=torch.uint8, device="cuda")
    scales = torch.empty((300,), dtype=torch.float32, device="cuda")
    runtime.quantize_fp8_rows(xt, codes, scales)
    torch.cuda.synchronize()
    oc, os_ = oracle.quantize_fp8_token(x)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), oc)


def _run_group(wl, layers=None, out_dtype=csa2.DTYPE_F32, scale=None):
    r = runtime.GroupRunner(wl, out_dtype=out_dtype, softmax_scale=scale, layers=layers)
    r.run()
    torch.cuda.synchronize()
    return r


def _check_caches(r, wl, seqs):
    kv = r.kv.cpu().numpy()
    kc = r.k_codes.cpu().numpy()
    ks = r.k_scales.cpu().numpy()
    starts = r.seq_start.cpu().numpy()
    for b, os_ in seqs.items():
        s0, n = int(starts[b]), wl.n_entries[b]
        assert np.array_equal(kv[s0:s0 + n], os_.kv_rows)
        assert np.array_equal(kc[s0:s0 + n], os_.k_codes)
        assert np.array_equal(ks[s0:s0 + n], os_.k_scales)


def _check_rows(r, wl, rows, check_attn=True):
    seqs = {}
    for row in rows:
        b, t = divmod(row, wl.T)
        if b not in seqs:
            seqs[b] = OracleSeq(wl, b)
        os_ = seqs[b]
        sel = os_.indices(t, r.modes)
        for l in range(len(r.modes)):
            idx, cnt = sel[l]
            got = r.layer_data[l]["idx"][row].cpu().numpy()
            assert np.array_equal(got, idx), f"layer {l} row {row}: index set differs"
            if check_attn:
                out, lse = os_.attention(l, t, idx, r.softmax_scale)
                g_out = r.layer_data[l]["out"][row].float().cpu().numpy()
                check_attention(g_out, out, f"layer {l} row {row}")
                g_lse = r.layer_data[l]["lse"][row].cpu().numpy()
                fin = np.isfinite(lse)
                assert np.array_equal(np.isfinite(g_lse), fin)
                assert np.all(np.abs(g_lse[fin] - lse[fin]) <= 1e-3)
    return seqs


def test_config0_tiny_full_layer():
    wl = synth.workload(0)
    r = _run_group(wl)
    seqs = _check_rows(r, wl, [0])
    _check_caches(r, wl, seqs)


@pytest.mark.parametrize("scale", [None, 1.0])
def test_ragged_batch_full_reuse(scale):
    wl = synth.scaled(synth.workload(1), B=4, n=[1000, 0, 37, 4500], K=64, H=32,
                      name="ragged_full_reuse")
    r = _run_group(wl, layers=3, scale=scale)
    seqs = _check_rows(r, wl, range(4))
    _check_caches(r, wl, seqs)
    # Reuse layers select exactly what the Full layer selected
    for l in (1, 2):
        assert torch.equal(r.layer_data[l]["idx"], r.layer_data[0]["idx"])
    # the empty sequence with an empty window gives zeros and lse = -inf
    assert not r.layer_data[0]["out"][1].any()


def test_reindex_group_scaled():
    wl = synth.scaled(synth.workload(2), B=3, n=[3000, 5000, 700], K=128, P=1000,
                      name="reindex_scaled")
    r = _run_group(wl)
    _check_rows(r, wl, range(3))


def test_long_rows_scaled():
    wl = synth.scaled(synth.workload(3), B=2, n=[70000, 41000], K=512, name="long_scaled")
    r = _run_group(wl, layers=2)
    _check_rows(r, wl, range(2))


def test_prefill_scaled():
    wl = synth.scaled(synth.workload(4), n=2000, T=96, K=256, name="prefill_scaled")
    r = _run_group(wl)
    _check_rows(r, wl, [0, 1, 2, 3, 47, 95])
    # causal: no selected entry lies beyond the query's visible range
    nv = [oracle.visible_entries(int(p), wl.n_entries[0]) for p in wl.q_pos(0)]
    idx = r.layer_data[0]["idx"].cpu().numpy()
    for t in range(wl.T):
        assert idx[t].max() < nv[t]


def test_bf16_output():
    wl = synth.scaled(synth.workload(1), B=2, n=3000, K=128, name="bf16_out")
    r = _run_group(wl, layers=1, out_dtype=csa2.DTYPE_BF16)
    for row in range(2):
        os_ = OracleSeq(wl, row)
        idx, _ = os_.indices(0, r.modes)[0]
        out, _ = os_.attention(0, 0, idx, r.softmax_scale)
        ref = torch.from_numpy(out).float().to(torch.bfloat16).float().numpy()
        got = r.layer_data[0]["out"][row].float().cpu().numpy()
        # bf16 rounding of the output itself is ~2^-9 relative; compare to the rounded reference
        assert np.linalg.norm(got - ref) <= 4e-3 * np.linalg.norm(ref)


def test_layer_events_same_result():
    """Per-layer ready/done events (csa2_layer_desc) only order work: the group's outputs with a
    side stream feeding each layer's query are bit-identical to a plain call."""
    wl = synth.scaled(synth.workload(2), B=3, n=5000, K=256, P=1200, name="events")
    r = _run_group(wl)
    ref = [ld["out"].clone() for ld in r.layer_data]
    host_q = [ld["q"].cpu().pin_memory() for ld in r.layer_data]
    for ld in r.layer_data:
        ld["q"].zero_()
        ld["out"].zero_()
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    ready = [torch.cuda.Event() for _ in r.modes]
    done = [torch.cuda.Event() for _ in r.modes]
    for ev in ready + done:
        ev.record(cur)
    torch.cuda.synchronize()
    r.set_layer_events([e.cuda_event for e in ready], [e.cuda_event for e in done])
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        for l, ld in enumerate(r.layer_data):
            ld["q"].copy_(host_q[l], non_blocking=True)
            ready[l].record(side)
    r.run()
    for l in range(len(r.modes)):
        done[l].synchronize()
    torch.cuda.synchronize()
    r.set_layer_events(None, None)
    for l, ld in enumerate(r.layer_data):
        assert torch.equal(ld["out"], ref[l]), l


def test_graph_replay_same_result():
    """The layer group captured in a CUDA graph and replayed gives the eager call's outputs."""
    wl = synth.scaled(synth.workload(2), B=3, n=4000, K=256, P=1000, name="graph")
    r = _run_group(wl)
    ref = [ld["out"].clone() for ld in r.layer_data]
    kernels = r.capture()
    assert kernels >= len(r.modes)
    for ld in r.layer_data:
        ld["out"].zero_()
    r.replay()
    torch.cuda.synchronize()
    for l, ld in enumerate(r.layer_data):
        assert torch.equal(ld["out"], ref[l]), l


@pytest.mark.parametrize("cfg,rows", [(1, [0, 17, 31]), (2, [0, 15]), (3, [0, 3]), (4, [0, 1000, 4095])])
def test_full_size_sampled(cfg, rows):
    """Full-size workloads in the bench's launch configuration; sampled rows vs the oracle."""
    wl = synth.workload(cfg)
    r = _run_group(wl)
    _check_rows(r, wl, rows)


def test_topk_heavy_ties_full_pool_reindex():
    """Selections where exact score ties straddle the K-th and P-th places.

    Keys of sequence 0 repeat with period 13, so its ~30000 scores take 13 values and the
    2048th and 3000th places fall inside tie classes; sequence 4 has zero head weights, so all
    of its scores are +0.  Ties are broken by entry index ascending ([A] section
    "压缩吸收注意力（二代）" orders the selection by score; the index order on ties is the
    reading both sides share).  Also: a distinct-key row with a ragged tail, a row with exactly
    K entries and an empty row.  Full mode emits the pool; a Reindex pass re-scores it with a
    second query.  Codes and scales are drawn directly (no quantisation step on either side).
    """
    rng = np.random.default_rng(4242)
    H_I, K, P = 8, 2048, 3000
    n = [30000, 4097, 2048, 0, 30000]
    B = len(n)
    starts = np.concatenate([[0], np.cumsum(n)[:-1]]).astype(np.int64)
    total = int(sum(n))
    kc = rng.integers(0, 256, (total, 32), dtype=np.uint8)
    ks = rng.integers(0x28, 0x49, (total, 4), dtype=np.uint8)
    base_c, base_s = kc[:13].copy(), ks[:13].copy()
    j = np.arange(n[0]) % 13
    kc[:n[0]], ks[:n[0]] = base_c[j], base_s[j]

    def query(seed):
        r = np.random.default_rng(seed)
        qc = r.integers(0, 256, (B, H_I, 32), dtype=np.uint8)
        qs = r.integers(0x28, 0x49, (B, H_I, 4), dtype=np.uint8)
        w = r.uniform(0, 1, (B, H_I)).astype(np.float32)
        w[2] = 0.0
        w[4] = 0.0
        return qc, qs, w

    dev = torch.device("cuda")
    g_kc, g_ks = torch.from_numpy(kc).to(dev), torch.from_numpy(ks).to(dev)
    g_start = torch.from_numpy(starts).to(dev)
    g_n = torch.tensor(n, dtype=torch.int32, device=dev)
    max_n = max(n)

    qc, qs, w = query(1)
    idx = torch.empty((B, K), dtype=torch.int32, device=dev)
    cnt = torch.empty((B,), dtype=torch.int32, device=dev)
    pool = torch.empty((B, P), dtype=torch.int32, device=dev)
    pool_len = torch.empty((B,), dtype=torch.int32, device=dev)
    ws = torch.empty(csa2.csa2_index_topk_workspace_size(csa2.MODE_FULL, B, max_n, K, P), dtype=torch.uint8,
                     device=dev)
    csa2.csa2_index_topk(csa2.MODE_FULL, torch.from_numpy(qc).to(dev), torch.from_numpy(qs).to(dev),
                         torch.from_numpy(w).to(dev), B, 1, H_I, g_kc, 32, g_ks, 4, g_start, g_n, max_n, None,
                         None, None, 0, K, idx, cnt, P, pool, pool_len, ws, ws.numel())
    torch.cuda.synchronize()
    o_pools = []
    for b in range(B):
        s0 = int(starts[b])
        oi, oc, op, opl, s = oracle.full_index(qc[b], qs[b], w[b], kc[s0:s0 + n[b]], ks[s0:s0 + n[b]], n[b], K, P)
        if b == 0:
            kth = np.sort(s)[::-1][K - 1]
            assert np.count_nonzero(s == kth) > 1 and np.count_nonzero(s > kth) < K   # a tie straddles K
        assert int(cnt[b]) == oc and np.array_equal(idx[b].cpu().numpy(), oi), f"top-K row {b}"
        assert int(pool_len[b]) == opl and np.array_equal(pool[b].cpu().numpy(), op), f"pool row {b}"
        o_pools.append((op, opl))
    assert np.array_equal(idx[4].cpu().numpy(), np.arange(K, dtype=np.int32))

    qc2, qs2, w2 = query(2)
    w2[4] = rng.uniform(0, 1, H_I).astype(np.float32)
    idx2 = torch.empty((B, K), dtype=torch.int32, device=dev)
    cnt2 = torch.empty((B,), dtype=torch.int32, device=dev)
    ws2 = torch.empty(csa2.csa2_index_topk_workspace_size(csa2.MODE_REINDEX, B, max_n, K, P), dtype=torch.uint8,
                      device=dev)
    csa2.csa2_index_topk(csa2.MODE_REINDEX, torch.from_numpy(qc2).to(dev), torch.from_numpy(qs2).to(dev),
                         torch.from_numpy(w2).to(dev), B, 1, H_I, g_kc, 32, g_ks, 4, g_start, g_n, max_n, None,
                         pool, pool_len, P, K, idx2, cnt2, 0, None, None, ws2, ws2.numel())
    torch.cuda.synchronize()
    for b in range(B):
        s0 = int(starts[b])
        op, opl = o_pools[b]
        oi, oc = oracle.reindex(qc2[b], qs2[b], w2[b], kc[s0:s0 + n[b]], ks[s0:s0 + n[b]], op, opl, K)
        assert int(cnt2[b]) == oc and np.array_equal(idx2[b].cpu().numpy(), oi), f"reindex row {b}"


@pytest.mark.parametrize("case", ["ragged_decode", "prefill"])
def test_step_writes_rewrite_identical_bytes(case):
    """A step's quantise-on-write (newest entry + indexer key per sequence, indexer queries, the
    step tokens' window entries) rewrites exactly the bytes the caches already hold, eagerly and
    inside a captured step, so the timed step reads the same caches and gives the same outputs."""
    if case == "ragged_decode":
        wl = synth.scaled(synth.workload(1), B=4, n=[1000, 0, 37, 4500], K=64, H=32, name="ragged_writes")
        r = _run_group(wl, layers=3)
    else:
        wl = synth.scaled(synth.workload(4), n=2000, T=96, K=256, name="prefill_writes")
        r = _run_group(wl)

    def snapshot():
        bufs = [r.kv, r.k_codes, r.k_scales, r.swa_codes_all, r.swa_scale_all.view(torch.int32)]
        bufs += [ld["iq_codes"] for ld in r.layer_data if "iq_codes" in ld]
        bufs += [ld["iq_scales"] for ld in r.layer_data if "iq_scales" in ld]
        bufs += [ld["out"].view(torch.int32) for ld in r.layer_data]
        bufs += [ld["idx"] for ld in r.layer_data]
        return [b.clone() for b in bufs]

    base = snapshot()
    r.step()
    torch.cuda.synchronize()
    for a, b in zip(base, snapshot()):
        assert torch.equal(a, b)
    r.capture(with_writes=True)
    r.replay()
    torch.cuda.synchronize()
    for a, b in zip(base, snapshot()):
        assert torch.equal(a, b)
