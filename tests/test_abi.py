"""The C-ABI library loads, exports every declared symbol, and validates arguments on the host.

No call here reaches the GPU: every case returns from argument validation before any launch.
"""
import ctypes
import os
import re
import subprocess

import pytest

import compressed_sparse_attention_quantize_b200 as csa2
from compressed_sparse_attention_quantize_b200 import build as csa2_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")

OK, INVALID, SHAPE, ALIGN, UNSUP, CUDA, TIMEOUT, WS, HOST = range(9)


@pytest.fixture(scope="module")
def L():
    csa2_build.build()
    return csa2.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"CSA2_API\s+[\w\s\*]*?\b(csa2_\w+)\s*\(", text)


def test_header_declares_the_four_calls():
    names = set(declared_functions())
    for n in ("csa2_quantize_kv", "csa2_index_topk", "csa2_sparse_attn", "csa2_layer_group"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    out = subprocess.check_output(["nm", "-D", "--defined-only", csa2.library_path()], text=True)
    exported = set(re.findall(r"\bT (csa2_\w+)", out))
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(L, n)


def test_status_strings(L):
    for s in range(9):
        assert csa2.csa2_status_string(s).startswith("CSA2")
    assert csa2.csa2_version() >= 1


def test_quantize_validation(L):
    q = L.csa2_quantize_kv
    # unknown format / dtype
    assert q(7, 16, 0, 4, 512, 512, 16, 256, 16, 32, None, None) == INVALID
    assert q(0, 16, 5, 4, 512, 512, 16, 256, 16, 32, None, None) == INVALID
    # dim not a multiple of 16, stride smaller than dim
    assert q(0, 16, 0, 4, 500, 512, 16, 256, 16, 32, None, None) == SHAPE
    assert q(0, 16, 0, 4, 512, 100, 16, 256, 16, 32, None, None) == SHAPE
    # rows == 0 is a no-op
    assert q(0, None, 0, 0, 512, 512, None, 256, None, 32, None, None) == OK
    assert q(0, None, 0, 0, 512, 1, None, 256, None, 32, None, None) == OK   # empty tensor strides
    # NULL input with rows > 0
    assert q(0, None, 0, 4, 512, 512, 16, 256, 16, 32, None, None) == INVALID
    # FP8 scales must be 4-byte aligned
    assert q(1, 16, 0, 4, 512, 512, 16, 512, 18, 4, None, None) == ALIGN


def test_compress_validation(L):
    c = L.csa2_compress_quantize_kv
    # x, dtype, entries, ratio, dim, x_stride, w, w_stride, codes, code_stride, scales, scale_stride, dst, stream
    assert c(16, 5, 4, 4, 512, 512, None, 0, 16, 256, 16, 32, None, None) == INVALID      # dtype
    assert c(None, 0, 0, 4, 512, 512, None, 0, None, 256, None, 32, None, None) == OK      # entries == 0
    assert c(16, 0, -1, 4, 512, 512, None, 0, 16, 256, 16, 32, None, None) == SHAPE
    assert c(16, 0, 4, 0, 512, 512, None, 0, 16, 256, 16, 32, None, None) == SHAPE        # ratio < 1
    assert c(16, 0, 4, 65, 512, 512, None, 0, 16, 256, 16, 32, None, None) == SHAPE       # ratio > max
    assert c(16, 0, 4, 4, 500, 512, None, 0, 16, 256, 16, 32, None, None) == SHAPE        # dim % 16
    assert c(16, 0, 4, 4, 512, 511, None, 0, 16, 256, 16, 32, None, None) == SHAPE        # x_stride
    assert c(16, 0, 4, 4, 512, 512, 16, 3, 16, 256, 16, 32, None, None) == SHAPE          # w_stride < m
    assert c(16, 0, 4, 4, 512, 512, None, 0, 16, 255, 16, 32, None, None) == SHAPE        # code_stride
    assert c(16, 0, 4, 4, 512, 512, None, 0, 16, 256, 16, 31, None, None) == SHAPE        # scale_stride
    assert c(None, 0, 4, 4, 512, 512, None, 0, 16, 256, 16, 32, None, None) == INVALID    # NULL x


def _attn(L, **kw):
    a = dict(q=16, B=1, T=1, H=64, D=512, kv=16, kv_row_stride=288, seq_start=16, n_entries=None, idx=16, cnt=None,
             K=64, swa_codes=16, swa_scale=16, swa_cap=128, swa_start=None, swa_len=16,
             softmax_scale=1.0, out=16, out_dtype=0, lse=None, workspace=16, ws_bytes=1 << 40,
             stream=None)
    a.update(kw)
    return L.csa2_sparse_attn(a["q"], a["B"], a["T"], a["H"], a["D"], a["kv"], a["kv_row_stride"],
                              a["seq_start"], a["n_entries"], a["idx"], a["cnt"], a["K"], a["swa_codes"],
                              a["swa_scale"],
                              a["swa_cap"], a["swa_start"], a["swa_len"], ctypes.c_float(a["softmax_scale"]),
                              a["out"], a["out_dtype"], a["lse"], a["workspace"], a["ws_bytes"], a["stream"])


def test_attn_validation(L):
    assert _attn(L, D=256) == UNSUP
    assert _attn(L, H=24) == SHAPE
    assert _attn(L, K=0) == SHAPE
    assert _attn(L, K=5000) == SHAPE
    assert _attn(L, kv=24) == ALIGN
    assert _attn(L, kv_row_stride=300) == ALIGN
    assert _attn(L, q=None) == INVALID
    assert _attn(L, out_dtype=9) == INVALID
    assert _attn(L, workspace=None) == WS
    assert _attn(L, ws_bytes=10) == WS


def test_workspace_queries():
    assert csa2.csa2_sparse_attn_workspace_size(32, 64, 2048) > 0
    assert csa2.csa2_index_topk_workspace_size(0, 32, 32768, 2048, 0) > 0
    assert csa2.csa2_index_topk_workspace_size(1, 16, 65536, 2048, 16000) > 0


def _group(modes, P=0):
    g = csa2.GroupDesc()
    g.B, g.T, g.H, g.D, g.H_I, g.K, g.P = 2, 1, 64, 512, 8, 64, P
    g.kv, g.kv_row_stride = 16, 288
    g.k_codes, g.k_code_stride, g.k_scales, g.k_scale_stride = 16, 32, 16, 4
    g.seq_start, g.n_entries, g.max_n = 16, 16, 1000
    g.swa_cap, g.swa_len = 128, 16
    g.softmax_scale = 1.0
    layers = []
    for m in modes:
        Ld = csa2.LayerDesc()
        Ld.mode = m
        Ld.q, Ld.iq_codes, Ld.iq_scales, Ld.iw, Ld.swa_codes, Ld.swa_scale, Ld.out = (16,) * 7
        layers.append(Ld)
    return g, layers


def test_layer_group_mode_table_validation(L):
    F, I, U = csa2.MODE_FULL, csa2.MODE_REINDEX, csa2.MODE_REUSE
    g, layers = _group([U, F])
    with pytest.raises(csa2.CSA2Error, match="INVALID_ARG"):
        csa2.csa2_layer_group_workspace_size(g, layers)
    g, layers = _group([F, I])          # Reindex needs a pool
    with pytest.raises(csa2.CSA2Error, match="INVALID_ARG"):
        csa2.csa2_layer_group_workspace_size(g, layers)
    g, layers = _group([F, I, U], P=300)
    assert csa2.csa2_layer_group_workspace_size(g, layers) > 0
    g, layers = _group([F, 7])
    with pytest.raises(csa2.CSA2Error, match="INVALID_ARG"):
        csa2.csa2_layer_group_workspace_size(g, layers)
    # too-small workspace is refused before anything is launched
    g, layers = _group([F, U])
    arr = (csa2.LayerDesc * 2)(*layers)
    assert L.csa2_layer_group(ctypes.byref(g), arr, 2, 16, 8, None) == WS


def test_layer_group_kept_pool_validation(L):
    F, I, U = csa2.MODE_FULL, csa2.MODE_REINDEX, csa2.MODE_REUSE
    g, layers = _group([F, I, U], P=300)
    base = csa2.csa2_layer_group_workspace_size(g, layers)
    g.pool_keep, g.pool_keep_len, g.pool_keep_n, g.max_new = 16, 16, 16, 64
    # the Reindex candidates grow by max_new, and so does the workspace
    assert csa2.csa2_layer_group_workspace_size(g, layers) > base
    g.max_new = -1
    with pytest.raises(csa2.CSA2Error, match="SHAPE"):
        csa2.csa2_layer_group_workspace_size(g, layers)
    g.max_new = 32768 - 300 + 1
    with pytest.raises(csa2.CSA2Error, match="SHAPE"):
        csa2.csa2_layer_group_workspace_size(g, layers)
    g.max_new = 64
    g.pool_keep_n = None
    with pytest.raises(csa2.CSA2Error, match="INVALID_ARG"):
        csa2.csa2_layer_group_workspace_size(g, layers)
    g.pool_keep_n, g.q_pos = 16, 16                 # decode only
    with pytest.raises(csa2.CSA2Error, match="INVALID_ARG"):
        csa2.csa2_layer_group_workspace_size(g, layers)
    # without Reindex layers the kept-pool fields are ignored
    g, layers = _group([F, U])
    g.pool_keep, g.max_new = 16, -5
    assert csa2.csa2_layer_group_workspace_size(g, layers) > 0


def test_pool_extend_validation(L):
    pe = L.csa2_pool_extend
    assert pe(None, 16, 10, 16, 16, None, 2, 1, 20, 16, 16, None) == INVALID
    assert pe(16, 16, 10, 16, 16, None, 0, 1, 20, 16, 16, None) == SHAPE
    assert pe(16, 16, -1, 16, 16, None, 2, 1, 20, 16, 16, None) == SHAPE
    assert pe(16, 16, 10, 16, 16, None, 2, 1, 0, 16, 16, None) == SHAPE
    assert pe(16, 16, 10, 16, 16, None, 2, 1, 32769, 16, 16, None) == SHAPE


def test_attention_plan_invariants():
    """The split plan covers the K + window keys with no empty split, in whole 128-key tiles,
    and the workspace query holds exactly one partial per (row, head group, split)."""
    part = (2 * 64 + 64 * 512) * 4
    for rows in (1, 3, 32, 148, 149, 1000, 4096):
        for H in (16, 32, 64, 128):
            for K in (1, 64, 2048, 4096):
                hg, sp, kps = csa2.csa2_sparse_attn_plan(rows, H, K)
                keys = K + 128
                assert hg == -(-H // 64)
                assert kps > 0 and kps % 128 == 0 and sp >= 1
                assert sp * kps >= keys and (sp - 1) * kps < keys, (rows, H, K, sp, kps)
                ws = csa2.csa2_sparse_attn_workspace_size(rows, H, K)
                assert ws == (256 if sp == 1 else rows * hg * sp * part + 256), (rows, H, K)
    # few rows split the keys finely; enough rows to fill the SMs take one split
    assert csa2.csa2_sparse_attn_plan(1, 64, 2048)[1] > csa2.csa2_sparse_attn_plan(64, 64, 2048)[1]
    assert csa2.csa2_sparse_attn_plan(4096, 64, 2048)[1] == 1


def test_attention_plan_validation():
    with pytest.raises(csa2.CSA2Error):
        csa2.csa2_sparse_attn_plan(0, 64, 2048)
    with pytest.raises(csa2.CSA2Error):
        csa2.csa2_sparse_attn_plan(32, 64, 0)


def test_default_plan_of_the_headline_decode_exceeds_the_noalloc_array():
    """32 rows x 64 heads x top-2048 (the 128K decode workload): the default split plan's
    partials need more than the 20 MiB array of csa2_sparse_attn_noalloc, so that call must
    (and does, on the GPU: tests/test_zz_no_alloc.py) run a plan fitted to the array."""
    hg, sp, kps = csa2.csa2_sparse_attn_plan(32, 64, 2048)
    assert sp > 1
    assert csa2.csa2_sparse_attn_workspace_size(32, 64, 2048) > (20 << 20)


def test_noalloc_validation(L):
    def call(**kw):
        a = dict(q=16, B=1, T=1, H=64, D=512, kv=16, kv_row_stride=288, seq_start=16, n_entries=None,
                 idx=16, cnt=None, K=64, swa_codes=16, swa_scale=16, swa_cap=128, swa_start=None,
                 swa_len=16, softmax_scale=1.0, out=16, out_dtype=0, lse=None, stream=None)
        a.update(kw)
        return L.csa2_sparse_attn_noalloc(
            a["q"], a["B"], a["T"], a["H"], a["D"], a["kv"], a["kv_row_stride"], a["seq_start"],
            a["n_entries"], a["idx"], a["cnt"], a["K"], a["swa_codes"], a["swa_scale"], a["swa_cap"],
            a["swa_start"], a["swa_len"], ctypes.c_float(a["softmax_scale"]), a["out"], a["out_dtype"],
            a["lse"], a["stream"])
    assert call(D=256) == UNSUP
    assert call(H=24) == SHAPE
    assert call(K=5000) == SHAPE
    assert call(kv=24) == ALIGN
    assert call(q=None) == INVALID


def test_quantize_batch_validation(L):
    J = csa2.QuantJob
    ok = csa2.quant_job(0, 16, 0, 4, 512, 512, 16, 256, 16, 32)
    bad = csa2.quant_job(0, 16, 0, 4, 500, 512, 16, 256, 16, 32)          # dim % 16
    arr = (J * 2)(ok, bad)
    assert L.csa2_quantize_kv_batch(arr, 2, None) == SHAPE               # nothing launched
    assert L.csa2_quantize_kv_batch(arr, 17, None) == SHAPE              # too many jobs
    assert L.csa2_quantize_kv_batch(None, 1, None) == INVALID
    assert L.csa2_quantize_kv_batch(None, 0, None) == OK
    empty = csa2.quant_job(0, None, 0, 0, 512, 512, None, 256, None, 32)
    assert L.csa2_quantize_kv_batch((J * 1)(empty), 1, None) == OK        # rows == 0 only


def test_host_alloc_validation(L):
    """csa2_host_alloc / csa2_host_free argument checks (none of them maps or registers memory)."""
    p = ctypes.c_void_p(1234)
    assert L.csa2_host_alloc(1 << 20, None) == INVALID
    assert L.csa2_host_alloc(0, ctypes.byref(p)) == SHAPE
    assert p.value is None                                   # *ptr cleared on every error
    assert L.csa2_host_alloc((1 << 40) + 1, ctypes.byref(p)) == SHAPE
    assert L.csa2_host_free(None) == OK
    assert L.csa2_host_free(ctypes.c_void_p(4096)) == INVALID  # not from csa2_host_alloc
