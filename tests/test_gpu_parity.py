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


def _e4m3_values():
    return np.array([oracle.e4m3_value(c) for c in range(0x7F)], np.float64)


def _nudge(x, steps):
    """x moved by `steps` fp32 ulps (elementwise, towards +inf for positive steps)."""
    x = x.astype(np.float32)
    for k in range(int(np.abs(steps).max(initial=0))):
        up = steps > k
        dn = steps < -k
        x = np.where(up, np.nextafter(x, np.float32(np.inf)), x)
        x = np.where(dn, np.nextafter(x, np.float32(-np.inf)), x)
    return x.astype(np.float32)


def _fp8_tie_rows(rng, rows, dim, exps=(-40, 40)):
    """Rows whose values sit on, or a few fp32 ulps from, mu * s for E4M3 midpoints mu, where
    s = amax/448 is the row's fp32 scale (amax near 2^e, e drawn from `exps`): the codes then
    depend on the exact quotient."""
    v = _e4m3_values()
    mids = 0.5 * (v[:-1] + v[1:])
    x = np.empty((rows, dim), np.float32)
    for r in range(rows):
        amax = np.float32(rng.uniform(1.0, 2.0) * 2.0 ** rng.integers(*exps))
        s = np.float32(amax / np.float32(448.0))
        mu = rng.choice(mids, dim)
        x[r] = _nudge(np.float32(mu * np.float64(s)), rng.integers(-2, 3, dim))
        x[r] *= np.where(rng.random(dim) < 0.5, -1, 1).astype(np.float32)
        x[r, rng.integers(dim)] = amax
    return x


def _fp4_tie_rows(rng, rows, dim):
    """Rows whose 16-channel blocks hold 6s (so the block scale is the E4M3 value s) and values
    on, or a few ulps from, mu * s for the E2M1 midpoints mu."""
    v = _e4m3_values()
    s_all = v[(v > 0) & (v <= 64)]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    x = np.empty((rows, dim), np.float32)
    for r in range(rows):
        for b in range(dim // 16):
            s = rng.choice(s_all)
            blk = _nudge(np.float32(rng.choice(mids, 16) * s), rng.integers(-2, 3, 16))
            blk *= np.where(rng.random(16) < 0.5, -1, 1).astype(np.float32)
            blk[rng.integers(16)] = np.float32(6.0 * s)
            x[r, b * 16:(b + 1) * 16] = blk
    return x


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_fp4_bitexact(dtype):
    rng = np.random.default_rng(100)
    x = _special_rows(rng, 777, 512)
    x[100:160] = _fp4_tie_rows(rng, 60, 512)
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


def test_quantize_batch_bitexact():
    """csa2_quantize_kv_batch: FP4 (f32 and bf16, 512- and 64-wide, scattered rows) and FP8 window
    jobs in one launch, each bit-exact vs the oracle; an empty job is skipped."""
    rng = np.random.default_rng(103)
    x4 = _special_rows(rng, 777, 512)
    x4b = torch.from_numpy(_special_rows(rng, 100, 512)).cuda().to(torch.bfloat16)
    xk = rng.standard_normal((50, 64)).astype(np.float32)
    x8 = _special_rows(rng, 300, 512)
    dst_k = torch.from_numpy(rng.permutation(80)[:50].astype(np.int64)).cuda()
    dst_8 = torch.from_numpy(rng.permutation(400)[:300].astype(np.int64)).cuda()
    kv = torch.zeros((777, 288), dtype=torch.uint8, device="cuda")
    kvb = torch.zeros((100, 288), dtype=torch.uint8, device="cuda")
    kc = torch.zeros((80, 32), dtype=torch.uint8, device="cuda")
    ks = torch.zeros((80, 4), dtype=torch.uint8, device="cuda")
    c8 = torch.zeros((400, 512), dtype=torch.uint8, device="cuda")
    s8 = torch.zeros((400,), dtype=torch.float32, device="cuda")
    g4, gk, g8 = torch.from_numpy(x4).cuda(), torch.from_numpy(xk).cuda(), torch.from_numpy(x8).cuda()
    jobs = [csa2.quant_job(csa2.FMT_FP4, g4, csa2.DTYPE_F32, 777, 512, 512, kv, 288, kv[:, 256:], 288),
            csa2.quant_job(csa2.FMT_FP8_TOKEN, g8, csa2.DTYPE_F32, 300, 512, 512, c8, 512, s8, 4, dst_8),
            csa2.quant_job(csa2.FMT_FP4, g4, csa2.DTYPE_F32, 0, 512, 512, kv, 288, kv[:, 256:], 288),
            csa2.quant_job(csa2.FMT_FP4, x4b, csa2.DTYPE_BF16, 100, 512, 512, kvb, 288, kvb[:, 256:], 288),
            csa2.quant_job(csa2.FMT_FP4, gk, csa2.DTYPE_F32, 50, 64, 64, kc, 32, ks, 4, dst_k)]
    csa2.csa2_quantize_kv_batch(jobs)
    torch.cuda.synchronize()
    oc, os_ = oracle.quantize_fp4(x4)
    assert np.array_equal(kv.cpu().numpy(), np.concatenate([oc, os_], axis=1))
    oc, os_ = oracle.quantize_fp4(x4b.float().cpu().numpy())
    assert np.array_equal(kvb.cpu().numpy(), np.concatenate([oc, os_], axis=1))
    oc, os_ = oracle.quantize_fp4(xk)
    d = dst_k.cpu().numpy()
    assert np.array_equal(kc.cpu().numpy()[d], oc) and np.array_equal(ks.cpu().numpy()[d], os_)
    oc, os_ = oracle.quantize_fp8_token(x8)
    d = dst_8.cpu().numpy()
    assert np.array_equal(c8.cpu().numpy()[d], oc)
    assert np.array_equal(s8.cpu().numpy()[d].view(np.uint32), os_.view(np.uint32))


def test_quantize_batch_ties_layouts():
    """csa2_quantize_kv_batch on values at and next to the rounding midpoints, on row lengths
    that end inside a thread's channels or exceed what a thread group holds, on rows that are
    not 16-byte aligned (scalar loads) and code rows that are not 4-byte aligned (byte stores),
    and on FP8 rows whose scale is too small or too large for the reciprocal shortcut."""
    rng = np.random.default_rng(104)
    f4 = _fp4_tie_rows(rng, 64, 512)
    cases = []                                         # (fmt, x f32 [rows, dim], pad, code_pad)
    cases.append((csa2.FMT_FP4, f4, 0, 0))
    cases.append((csa2.FMT_FP4, _fp4_tie_rows(rng, 33, 64), 1, 1))
    for dim in (16, 528, 2048, 2064):
        cases.append((csa2.FMT_FP8_TOKEN, _fp8_tie_rows(rng, 9, dim), 0, 0))
    odd = np.concatenate([_fp8_tie_rows(rng, 4, 512, (-96, -94)),     # scales below 2^-100
                          _fp8_tie_rows(rng, 4, 512, (110, 113)),     # scales above 2^100
                          _fp8_tie_rows(rng, 4, 512, (-136, -126))])  # subnormal amax
    cases.append((csa2.FMT_FP8_TOKEN, odd, 3, 1))
    jobs, outs = [], []
    for fmt, x, pad, cpad in cases:
        rows, dim = x.shape
        if pad:                                        # rows start one element in: misaligned
            xp = np.zeros((rows, dim + pad + 1), np.float32)
            xp[:, 1:dim + 1] = x
            xt = torch.from_numpy(xp).cuda()
            xv = xt[:, 1:]
        else:
            xt = torch.from_numpy(np.ascontiguousarray(x)).cuda()
            xv = xt
        if fmt == csa2.FMT_FP4:
            cs = dim // 2 + dim // 16 + cpad
            buf = torch.zeros((rows + 3, cs), dtype=torch.uint8, device="cuda")
            dst = torch.from_numpy(rng.permutation(rows + 3)[:rows].astype(np.int64)).cuda()
            jobs.append(csa2.quant_job(fmt, xv, csa2.DTYPE_F32, rows, dim, xv.stride(0), buf, cs,
                                       buf[:, dim // 2:], cs, dst))
            outs.append((fmt, x, buf, dst, None))
        else:
            cs = dim + cpad
            buf = torch.zeros((rows + 3, cs), dtype=torch.uint8, device="cuda")
            sc = torch.zeros((rows + 3,), dtype=torch.float32, device="cuda")
            dst = torch.from_numpy(rng.permutation(rows + 3)[:rows].astype(np.int64)).cuda()
            jobs.append(csa2.quant_job(fmt, xv, csa2.DTYPE_F32, rows, dim, xv.stride(0), buf, cs, sc, 4, dst))
            outs.append((fmt, x, buf, dst, sc))
        outs[-1] = outs[-1] + (xt,)
    csa2.csa2_quantize_kv_batch(jobs)
    torch.cuda.synchronize()
    for fmt, x, buf, dst, sc, _ in outs:
        d = dst.cpu().numpy()
        dim = x.shape[1]
        got = buf.cpu().numpy()[d]
        if fmt == csa2.FMT_FP4:
            oc, os_ = oracle.quantize_fp4(x)
            assert np.array_equal(got[:, :dim // 2], oc), dim
            assert np.array_equal(got[:, dim // 2:dim // 2 + dim // 16], os_), dim
        else:
            oc, os_ = oracle.quantize_fp8_token(x)
            assert np.array_equal(got[:, :dim], oc), dim
            assert np.array_equal(sc.cpu().numpy()[d].view(np.uint32), os_.view(np.uint32)), dim


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
    x[20:60] = _fp8_tie_rows(rng, 40, 512)
    x[60:64] = _fp8_tie_rows(rng, 4, 512, (-136, -94))    # scales below 2^-100
    x[64:68] = _fp8_tie_rows(rng, 4, 512, (110, 113))     # scales above 2^100
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


@pytest.mark.parametrize("R", [1, 3])
def test_pool_kept_across_decode_steps(R):
    """Kept candidate pool over consecutive decode steps: the context grows by a few entries per
    step (sequence 1 not at all), the pool is rebuilt every R steps and the Reindex layers
    search it plus the entries written since; every layer's selection at every step equals the
    oracle's decode_steps_with_pool."""
    n = [3000, 5000, 700]
    growth = [37, 0, 5]
    steps = 7
    wl = synth.scaled(synth.workload(2), B=3, n=n, K=128, P=600, name="pool_kept")
    r = runtime.GroupRunner(wl, layers=4)
    r.keep_pool(max_new=max(growth) * steps)
    n_steps = [[n[b] - (steps - 1 - s) * growth[b] for s in range(steps)] for b in range(3)]
    got = []
    for s in range(steps):
        r.n_entries.copy_(torch.tensor([n_steps[b][s] for b in range(3)], dtype=torch.int32))
        r.run(refresh=(s % R == 0))
        torch.cuda.synchronize()
        got.append([r.layer_data[l]["idx"].cpu().numpy().copy() for l in range(4)])
    assert csa2.csa2_device_error() == 0
    for b in range(3):
        os_ = OracleSeq(wl, b)
        inputs = [None if m == "U" else (os_.layer(l)["qc"][0], os_.layer(l)["qs"][0], os_.layer(l)["w"][0])
                  for l, m in enumerate(r.modes)]
        ref = oracle.decode_steps_with_pool(r.modes, [inputs] * steps, os_.k_codes, os_.k_scales,
                                            n_steps[b], wl.K, wl.P, R)
        for s in range(steps):
            for l in range(4):
                assert np.array_equal(got[s][l][b], ref[s][l][0]), f"step {s} layer {l} seq {b}"
    # attention of the last step reads the last step's selections
    os_ = OracleSeq(wl, 0)
    out, _ = os_.attention(1, 0, got[-1][1][0], r.softmax_scale)
    check_attention(r.layer_data[1]["out"][0].cpu().numpy(), out, "layer 1 seq 0")


def test_pool_extend_matches_oracle():
    rng = np.random.default_rng(11)
    B, T, P_in, P_out = 5, 3, 40, 70
    rows = B * T
    n_ref = np.array([0, 100, 500, 64, 9], np.int32)
    n_ent = n_ref + np.array([0, 29, 30, 3, 0], np.int32)
    pool = np.full((rows, P_in), -1, np.int32)
    plen = np.zeros(rows, np.int32)
    for r in range(rows):
        b = r // T
        k = int(rng.integers(0, min(P_in, n_ref[b]) + 1))
        pool[r, :k] = np.sort(rng.choice(max(n_ref[b], 1), size=k, replace=False)) if k else []
        plen[r] = k
    dev = torch.device("cuda")
    out = torch.full((rows, P_out), -7, dtype=torch.int32, device=dev)
    olen = torch.zeros(rows, dtype=torch.int32, device=dev)
    tp = [torch.from_numpy(x).to(dev) for x in (pool, plen, n_ref, n_ent)]
    csa2.csa2_pool_extend(tp[0], tp[1], P_in, tp[2], tp[3], None, B, T, P_out, out, olen)
    torch.cuda.synchronize()
    assert csa2.csa2_device_error() == 0
    out, olen = out.cpu().numpy(), olen.cpu().numpy()
    for r in range(rows):
        b = r // T
        ref = oracle.extend_pool(pool[r], plen[r], n_ref[b], n_ent[b])
        assert olen[r] == len(ref)
        assert np.array_equal(out[r, :len(ref)], ref)
        assert np.all(out[r, len(ref):] == -7)          # nothing written past the count


def test_pool_kept_overflow_flags_shape():
    """More new entries than max_new since the refresh: the device error word reads
    CSA2_ERR_SHAPE and the call still completes."""
    wl = synth.scaled(synth.workload(2), B=1, n=[2000], K=64, P=300, name="pool_overflow")
    r = runtime.GroupRunner(wl, layers=2)
    r.keep_pool(max_new=8)
    r.n_entries.fill_(1900)
    r.run(refresh=True)
    torch.cuda.synchronize()
    assert csa2.csa2_device_error() == 0
    r.n_entries.fill_(2000)
    r.run(refresh=False)
    torch.cuda.synchronize()
    assert csa2.csa2_device_error() == csa2.CSA2_ERR_SHAPE
    assert csa2.csa2_device_error() == 0


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


def _bf16_boundary_between(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """True where a rounding boundary of bf16 (the midpoint of two adjacent bf16 values) lies
    between a and b (inclusive), i.e. where round-to-nearest of a and of b may differ."""
    ta = torch.from_numpy(np.asarray(a, np.float32))
    tb = torch.from_numpy(np.asarray(b, np.float32))
    return (ta.to(torch.bfloat16) != tb.to(torch.bfloat16)).numpy()


def test_bf16_output():
    """bf16 output, elementwise.  (1) It is exactly the kernel's own fp32 result rounded to
    nearest-even bf16 (same launch plan, out_dtype fp32 vs bf16).  (2) Against the oracle's
    fp64 result rounded to bf16 it is equal wherever no bf16 rounding boundary lies between the
    oracle's value and the kernel's fp32 value; the elements where one does are counted
    (their difference comes from the fp32 kernel arithmetic, which the fp32 parity bound
    covers)."""
    wl = synth.scaled(synth.workload(1), B=2, n=3000, K=128, name="bf16_out")
    r16 = _run_group(wl, layers=1, out_dtype=csa2.DTYPE_BF16)
    r32 = _run_group(wl, layers=1, out_dtype=csa2.DTYPE_F32)
    boundary_cases = 0
    for row in range(2):
        got16 = r16.layer_data[0]["out"][row].cpu()
        got32 = r32.layer_data[0]["out"][row].cpu()
        assert torch.equal(got16, got32.to(torch.bfloat16)), f"row {row}: bf16 != rn(fp32)"
        os_ = OracleSeq(wl, row)
        idx, _ = os_.indices(0, r16.modes)[0]
        out, _ = os_.attention(0, 0, idx, r16.softmax_scale)
        check_attention(got32.numpy(), out, f"row {row} (fp32)")
        ref16 = torch.from_numpy(out.astype(np.float32)).to(torch.bfloat16)
        differ = (got16 != ref16).numpy()
        allowed = _bf16_boundary_between(out.astype(np.float32), got32.numpy())
        assert not (differ & ~allowed).any(), f"row {row}: bf16 differs with no rounding boundary in between"
        boundary_cases += int(differ.sum())
    print(f"bf16 output: {boundary_cases} of {2 * wl.H * 512} elements on the other side of a "
          f"rounding boundary from the oracle")


def test_layer_events_same_result():
    """Per-layer ready/attn_ready/done events (csa2_layer_desc) only order work: the group's
    outputs and selections with a side stream feeding each layer's indexer inputs (ready) and
    then its main query (attn_ready) are bit-identical to a plain call."""
    wl = synth.scaled(synth.workload(2), B=3, n=5000, K=256, P=1200, name="events")
    r = _run_group(wl)
    ref = [ld["out"].clone() for ld in r.layer_data]
    ref_idx = [ld["idx"].clone() for ld in r.layer_data]
    names = ("iq_codes", "iq_scales", "iw")
    host_q = [ld["q"].cpu().pin_memory() for ld in r.layer_data]
    host_i = [{k: ld[k].cpu().pin_memory() for k in names if k in ld} for ld in r.layer_data]
    for ld in r.layer_data:
        for k in ("q", "out", "idx") + names:
            if k in ld:
                ld[k].zero_()
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    ready = [torch.cuda.Event() for _ in r.modes]
    attn_ready = [torch.cuda.Event() for _ in r.modes]
    done = [torch.cuda.Event() for _ in r.modes]
    for ev in ready + attn_ready + done:
        ev.record(cur)
    torch.cuda.synchronize()
    r.set_layer_events([e.cuda_event for e in ready], [e.cuda_event for e in done],
                       [e.cuda_event for e in attn_ready])
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        for l, ld in enumerate(r.layer_data):
            for k, h in host_i[l].items():
                ld[k].copy_(h, non_blocking=True)
            ready[l].record(side)
            ld["q"].copy_(host_q[l], non_blocking=True)
            attn_ready[l].record(side)
    r.run()
    for l in range(len(r.modes)):
        done[l].synchronize()
    torch.cuda.synchronize()
    r.set_layer_events(None, None)
    for l, ld in enumerate(r.layer_data):
        assert torch.equal(ld["out"], ref[l]), l
        assert torch.equal(ld["idx"], ref_idx[l]), l


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


@pytest.mark.parametrize("long_rows", [False, True])
def test_topk_heavy_ties_full_pool_reindex(long_rows):
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
    # long_rows: rows beyond what one CTA holds in shared memory, so every chunk of a row selects
    # first and the union is selected again (tie classes then cross chunk boundaries)
    n = [100000, 4097, 2048, 0, 70000] if long_rows else [30000, 4097, 2048, 0, 30000]
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


def test_header_limits_group():
    """Every size limit of the header in one Full, Reindex, Reuse group: H = CSA2_MAX_HEADS (128,
    two head groups of 64), H_I = CSA2_MAX_INDEX_HEADS (16, 64 MMA columns in the indexer),
    K = CSA2_MAX_TOPK (4096) and P = CSA2_MAX_POOL (32768, a pool smaller than the rows)."""
    wl = synth.scaled(synth.workload(2), B=2, n=[40000, 33000], K=4096, P=32768, H=128, HI=16,
                      modes=("F", "I", "U"), name="limits")
    r = _run_group(wl)
    _check_rows(r, wl, range(2))


def _random_key_cache(rng, n):
    starts = np.concatenate([[0], np.cumsum(n)[:-1]]).astype(np.int64)
    total = int(sum(n))
    kc = rng.integers(0, 256, (total, 32), dtype=np.uint8)
    ks = rng.integers(0x20, 0x50, (total, 4), dtype=np.uint8)
    return starts, kc, ks


@pytest.mark.parametrize("K,P", [(2048, 16000), (4096, 32768)])
def test_select_rows_beyond_cluster_capacity(K, P):
    """Rows longer than an 8-CTA cluster holds (262,144 candidates) take the one-CTA radix select:
    a row of 262,145 entries and one of 300,000, top-K and pool bit-exact vs the oracle, then a
    Reindex of that pool."""
    rng = np.random.default_rng(5150 + K)
    H_I = 8
    n = [262145, 300000]
    B = len(n)
    starts, kc, ks = _random_key_cache(rng, n)
    dev = torch.device("cuda")
    g_kc, g_ks = torch.from_numpy(kc).to(dev), torch.from_numpy(ks).to(dev)
    g_start = torch.from_numpy(starts).to(dev)
    g_n = torch.tensor(n, dtype=torch.int32, device=dev)
    max_n = max(n)

    def query(seed):
        q = np.random.default_rng(seed)
        return (q.integers(0, 256, (B, H_I, 32), dtype=np.uint8), q.integers(0x28, 0x49, (B, H_I, 4), dtype=np.uint8),
                q.uniform(0, 1, (B, H_I)).astype(np.float32))

    qc, qs, w = query(11)
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
    pools = []
    for b in range(B):
        s0 = int(starts[b])
        oi, oc, op, opl, _ = oracle.full_index(qc[b], qs[b], w[b], kc[s0:s0 + n[b]], ks[s0:s0 + n[b]], n[b], K, P)
        assert int(cnt[b]) == oc and np.array_equal(idx[b].cpu().numpy(), oi), f"top-K row {b}"
        assert int(pool_len[b]) == opl and np.array_equal(pool[b].cpu().numpy(), op), f"pool row {b}"
        pools.append((op, opl))
    qc2, qs2, w2 = query(12)
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
        op, opl = pools[b]
        oi, oc = oracle.reindex(qc2[b], qs2[b], w2[b], kc[s0:s0 + n[b]], ks[s0:s0 + n[b]], op, opl, K)
        assert int(cnt2[b]) == oc and np.array_equal(idx2[b].cpu().numpy(), oi), f"reindex row {b}"


def test_attention_contract_checks():
    """Ids, window slots and counts outside csa2_sparse_attn's caller contract are caught on the
    device: the key is skipped (or the count clamped), the device error word says which, and the
    other rows are unaffected.  Every injected value still points inside the caller's buffers
    (sequence 0 is not the last one), so even a missing check would read valid memory."""
    wl = synth.scaled(synth.workload(1), B=2, n=[3000, 2500], K=256, name="contract")
    r = _run_group(wl, layers=1)
    assert csa2.csa2_device_error() == 0
    ld = r.layer_data[0]
    idx = ld["idx"].clone()
    cnt = (idx >= 0).sum(dim=1).to(torch.int32)
    ws_bytes = csa2.csa2_sparse_attn_workspace_size(r.rows, wl.H, wl.K)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device="cuda")

    def attn(idx_, cnt_, swa_start=None, swa_len=None):
        out = torch.full((r.rows, wl.H, 512), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.empty((r.rows, wl.H), dtype=torch.float32, device="cuda")
        csa2.csa2_sparse_attn(ld["q"], wl.B, wl.T, wl.H, 512, r.kv, 288, r.seq_start, r.n_entries, idx_, cnt_,
                              wl.K, ld["swa_codes"], ld["swa_scale"], r.swa_cap,
                              r.swa_start if swa_start is None else swa_start,
                              r.swa_len if swa_len is None else swa_len, r.softmax_scale, out, csa2.DTYPE_F32,
                              lse, ws, ws_bytes)
        torch.cuda.synchronize()
        return out

    clean = attn(idx, cnt)
    assert csa2.csa2_device_error() == 0
    # an id equal to sequence 0's entry count (it would read sequence 1's first row)
    bad = idx.clone()
    bad[0, 5] = wl.n_entries[0]
    out = attn(bad, cnt)
    assert csa2.csa2_device_error() == csa2.CSA2_ERR_INVALID_ARG
    assert csa2.csa2_device_error() == 0                       # read and cleared
    assert torch.equal(out[1], clean[1])
    skipped = idx[0].cpu().numpy().copy()
    skipped[5] = -1
    os_ = OracleSeq(wl, 0)
    ref, _ = os_.attention(0, 0, skipped, r.softmax_scale)
    check_attention(out[0].cpu().numpy(), ref, "row 0 with the bad id skipped")
    # a window that runs past the buffer (its last slot would be sequence 1's slot 0)
    st = r.swa_start.clone()
    st[0] = 1
    out = attn(idx, cnt, swa_start=st)
    assert csa2.csa2_device_error() == csa2.CSA2_ERR_INVALID_ARG
    assert torch.equal(out[1], clean[1])
    # a count above K and a window length above 128 are clamped
    big = cnt.clone()
    big[0] = wl.K + 7
    out = attn(idx, big)
    assert csa2.csa2_device_error() == csa2.CSA2_ERR_SHAPE
    assert torch.equal(out[0], clean[0]) and torch.equal(out[1], clean[1])
    long_win = r.swa_len.clone()
    long_win[1] = 200
    attn(idx, cnt, swa_len=long_win)
    assert csa2.csa2_device_error() == csa2.CSA2_ERR_SHAPE


@pytest.mark.parametrize("G", [1, 3])
def test_topk_merge_shards_matches_oracle(G):
    """csa2_topk_merge_shards on G scored lists (one list is selected in place) equals the oracle's
    top-K of their union: scores with ties, ragged list lengths (one empty), ids ascending."""
    rng = np.random.default_rng(77 + G)
    rows, K_in, K = 5, 6000, 2048
    scores = rng.integers(0, 900, (G, rows, K_in)).astype(np.float32) / np.float32(7)
    ids = np.zeros((G, rows, K_in), np.int32)
    cnt = rng.integers(1500, K_in + 1, (G, rows)).astype(np.int32)
    cnt[0, 3] = 0
    for g in range(G):
        for r in range(rows):
            ids[g, r] = np.sort(rng.choice(50000, K_in, replace=False)).astype(np.int32) + g * 50000
    dev = torch.device("cuda")
    out = torch.empty((rows, K), dtype=torch.int32, device=dev)
    oc = torch.empty((rows,), dtype=torch.int32, device=dev)
    ws = torch.empty(csa2.csa2_topk_merge_shards_workspace_size(G, rows, K_in), dtype=torch.uint8, device=dev)
    csa2.csa2_topk_merge_shards(torch.from_numpy(scores).to(dev), torch.from_numpy(ids).to(dev), None,
                                torch.from_numpy(cnt).to(dev), G, rows, K_in, K, out, oc, ws, ws.numel())
    torch.cuda.synchronize()
    for r in range(rows):
        s = np.concatenate([scores[g, r, :cnt[g, r]] for g in range(G)])
        i = np.concatenate([ids[g, r, :cnt[g, r]] for g in range(G)])
        ref, rc = oracle.topk(s, K, ids=i)
        assert int(oc[r]) == rc and np.array_equal(out[r].cpu().numpy(), ref), r


def test_host_buffers_copy_and_graph():
    """csa2_host_alloc buffers (through host_empty): page-locked, asynchronous copies both ways
    on a side stream and inside a CUDA graph return the bytes written; a second free of the
    same address is refused."""
    src = csa2.host_empty((1000, 512), torch.bfloat16)
    assert src.is_pinned()
    ref = torch.randn((1000, 512), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    src.copy_(ref)
    dst = csa2.host_empty((1000, 512), torch.bfloat16)
    dev = torch.empty((1000, 512), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dev.copy_(src, non_blocking=True)
        dev.mul_(2)
        dst.copy_(dev, non_blocking=True)
    s.synchronize()
    assert torch.equal(dst, ref * 2)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dev.copy_(src, non_blocking=True)
        dev.add_(1)
        dst.copy_(dev, non_blocking=True)
    src.copy_(ref * 3)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(dst, ref * 3 + 1)
    del g
    p = csa2.csa2_host_alloc(3 << 20)
    csa2.csa2_host_free(p)
    with pytest.raises(csa2.CSA2Error):
        csa2.csa2_host_free(p)
