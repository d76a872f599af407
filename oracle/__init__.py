"""CSA2 reference oracle: TEST INFRASTRUCTURE ONLY.

A plain CPU restatement of the CSA2 hot path (FP4/FP8 quantise-on-write,
indexer scoring, top-K, Full/Reindex/Reuse layer modes, attention over the
selected entries plus the sliding window).  The arithmetic lives in
``csa2_oracle.c``; this module loads it with ctypes and composes the layer
modes in plain Python.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline and
reference legs of ``bench.py`` may import this package.  It imports nothing
from the CUDA library and the library never imports it.

Sources (web pages about the DeepSeek V4.1 Flash report):
  [A] "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径"
  [B] "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型"

Every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py``.  Parity unpinned: the pool that ``full_index``
builds (the top-min(P, n) of the Full layer's own order) is pinned as that
reading (it holds the top-K; Reindex over the whole context gives the Full
selection), but the pages do not say how the model forms or refreshes its
pool, so nothing pins the reading itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.c")
_SO = os.path.join(_HERE, "libcsa2_oracle.so")

D_LATENT = 512     # main-KV latent width
D_INDEX = 64       # indexer key/query width
KV_ROW_BYTES = 288  # 256 B of E2M1 codes + 32 B of E4M3 scales per main entry

_lib = None

u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc, IEEE arithmetic, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-shared", "-fPIC", "-o", _SO, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e2m1_value.argtypes = [ctypes.c_int]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [ctypes.c_int]
        L.oracle_e2m1_encode.restype = ctypes.c_int
        L.oracle_e2m1_encode.argtypes = [ctypes.c_double]
        L.oracle_e4m3_encode.restype = ctypes.c_int
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_quantize_fp4.restype = None
        L.oracle_quantize_fp4.argtypes = [f32p, ctypes.c_int64, ctypes.c_int, u8p, u8p]
        L.oracle_compress_fp4.restype = None
        L.oracle_compress_fp4.argtypes = [f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_void_p, u8p, u8p]
        L.oracle_dequantize_fp4.restype = None
        L.oracle_dequantize_fp4.argtypes = [u8p, u8p, ctypes.c_int64, ctypes.c_int, f64p]
        L.oracle_quantize_fp8_token.restype = None
        L.oracle_quantize_fp8_token.argtypes = [f32p, ctypes.c_int64, ctypes.c_int, u8p, f32p]
        L.oracle_index_scores.restype = None
        L.oracle_index_scores.argtypes = [u8p, u8p, f32p, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_int64,
                                          ctypes.c_void_p, ctypes.c_int64,
                                          ctypes.c_void_p, ctypes.c_int64, f32p]
        L.oracle_topk.restype = ctypes.c_int32
        L.oracle_topk.argtypes = [f32p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, i32p]
        L.oracle_attention.restype = None
        L.oracle_attention.argtypes = [u16p, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                       i32p, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                       ctypes.c_double, f64p, f64p]
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_num_threads.argtypes = []
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().oracle_num_threads()


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------
def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def e2m1_encode(v: float) -> int:
    return lib().oracle_e2m1_encode(float(v))


def e4m3_encode(v: float) -> int:
    return lib().oracle_e4m3_encode(float(v))


# --------------------------------------------------------------------------
# quantisers
# --------------------------------------------------------------------------
def quantize_fp4(x: np.ndarray):
    """[B: FP4 量化 + Bounded Replay] E2M1 codes + one E4M3 scale per 16 channels.

    x: float32 [rows, dim] -> (codes uint8 [rows, dim/2], scales uint8 [rows, dim/16]).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, dim = x.shape
    assert dim % 16 == 0
    codes = np.empty((rows, dim // 2), np.uint8)
    scales = np.empty((rows, dim // 16), np.uint8)
    lib().oracle_quantize_fp4(x, rows, dim, codes, scales)
    return codes, scales


def compress_fp4(x: np.ndarray, ratio: int, w: np.ndarray = None):
    """[B: CSA2：三层压缩一次吃满] every `ratio` tokens -> one entry, as the weighted sum
    sum_i w[e, i] * x[ratio*e + i] in fp32 (token order, no fused multiply-add; w=None is the
    mean), then FP4-quantised like quantize_fp4.

    x: float32 [entries*ratio, dim]; w: float32 [entries, ratio] or None.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    tokens, dim = x.shape
    assert dim % 16 == 0 and tokens % ratio == 0
    entries = tokens // ratio
    wp = None
    if w is not None:
        w = np.ascontiguousarray(w, dtype=np.float32)
        assert w.shape == (entries, ratio)
        wp = w.ctypes.data
    codes = np.empty((entries, dim // 2), np.uint8)
    scales = np.empty((entries, dim // 16), np.uint8)
    lib().oracle_compress_fp4(x, entries, ratio, dim, wp, codes, scales)
    return codes, scales


def dequantize_fp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows = codes.shape[0]
    dim = codes.shape[1] * 2
    out = np.empty((rows, dim), np.float64)
    lib().oracle_dequantize_fp4(codes, scales, rows, dim, out)
    return out


def quantize_fp8_token(x: np.ndarray):
    """8-bit sliding-window rows: E4M3 codes with one fp32 scale (amax/448) per token."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, dim = x.shape
    codes = np.empty((rows, dim), np.uint8)
    scales = np.empty((rows,), np.float32)
    lib().oracle_quantize_fp8_token(x, rows, dim, codes, scales)
    return codes, scales


def pack_kv_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Main-KV rows as stored: 256 B of codes then 32 B of scales (288 B per entry)."""
    rows = codes.shape[0]
    out = np.empty((rows, KV_ROW_BYTES), np.uint8)
    out[:, :256] = codes
    out[:, 256:] = scales
    return out


# --------------------------------------------------------------------------
# indexer and top-K
# --------------------------------------------------------------------------
def index_scores(q_codes, q_scales, w, k_codes, k_scales, key_index=None) -> np.ndarray:
    """fp32 indexer score of one query row against keys (fixed summation order).

    q_codes [H,32] u8, q_scales [H,4] u8, w [H] f32, k_codes [n,32] u8, k_scales [n,4] u8.
    key_index: optional int32 list of key rows to score, in order.
    """
    q_codes = np.ascontiguousarray(q_codes, np.uint8)
    q_scales = np.ascontiguousarray(q_scales, np.uint8)
    w = np.ascontiguousarray(w, np.float32)
    k_codes = np.ascontiguousarray(k_codes, np.uint8)
    k_scales = np.ascontiguousarray(k_scales, np.uint8)
    H = q_codes.shape[0]
    if key_index is not None:
        key_index = np.ascontiguousarray(key_index, np.int32)
        n = key_index.shape[0]
        kip = key_index.ctypes.data
    else:
        n = k_codes.shape[0]
        kip = None
    out = np.empty((n,), np.float32)
    if n == 0:
        return out
    lib().oracle_index_scores(q_codes, q_scales, w, H,
                              k_codes.ctypes.data, k_codes.strides[0],
                              k_scales.ctypes.data, k_scales.strides[0],
                              kip, n, out)
    return out


def topk(scores: np.ndarray, K: int, ids: Optional[np.ndarray] = None):
    """[A: 压缩吸收注意力（二代）] top-K by (score desc, index asc).

    Returns (idx int32 [K] ascending, padded with -1; count)."""
    scores = np.ascontiguousarray(scores, np.float32)
    n = scores.shape[0]
    out = np.empty((max(K, 0),), np.int32)
    idp = None
    if ids is not None:
        ids = np.ascontiguousarray(ids, np.int32)
        idp = ids.ctypes.data
    cnt = lib().oracle_topk(scores if n else np.zeros(1, np.float32), idp, n, K, out)
    return out, int(cnt)


def full_index(q_codes, q_scales, w, k_codes, k_scales, n_vis: int, K: int, P: int = 0):
    """Full mode: score all visible entries, top-K, and (P > 0) the candidate pool.

    [A: 压缩吸收注意力（二代）]: after the first layer scans the context it keeps a
    candidate pool that later layers search.  Reading: the pool is the top-min(P, n)
    of the same order, which nests the top-K.  Which pool the model really builds is
    parity unpinned (the pages do not say how it is formed or refreshed).
    """
    s = index_scores(q_codes, q_scales, w, k_codes[:n_vis], k_scales[:n_vis])
    idx, cnt = topk(s, K)
    pool = pool_len = None
    if P > 0:
        pool, pool_len = topk(s, P)
    return idx, cnt, pool, pool_len, s


def reindex(q_codes, q_scales, w, k_codes, k_scales, pool: np.ndarray, pool_len: int, K: int):
    """Reindex mode ([B: CSA2：三层压缩一次吃满]): re-score only the pool with this
    layer's own indexer query and take top-K within it."""
    cand = np.ascontiguousarray(pool[:pool_len], np.int32)
    s = index_scores(q_codes, q_scales, w, k_codes, k_scales, key_index=cand)
    return topk(s, K, ids=cand)


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def attention(q_bf16: np.ndarray, kv_rows: np.ndarray, idx: np.ndarray,
              swa_codes: np.ndarray, swa_scale: np.ndarray, softmax_scale: float):
    """Attention of one query row over the selected main entries + its SWA window.

    q_bf16: uint16 [H, D] (bf16 bits); kv_rows: uint8 [n, 288] main entries;
    idx: int32 [K] (-1 = empty); swa_codes uint8 [w, D]; swa_scale float32 [w].
    Returns (out float64 [H, D], lse float64 [H]).
    """
    q = np.ascontiguousarray(q_bf16, np.uint16)
    H, D = q.shape
    assert D == D_LATENT
    kv = np.ascontiguousarray(kv_rows, np.uint8)
    idx = np.ascontiguousarray(idx, np.int32)
    swc = np.ascontiguousarray(swa_codes, np.uint8).reshape(-1, D)
    sws = np.ascontiguousarray(swa_scale, np.float32).reshape(-1)
    out = np.empty((H, D), np.float64)
    lse = np.empty((H,), np.float64)
    kvp = kv.ctypes.data if kv.size else None
    lib().oracle_attention(q, H, D, kvp, (kv.ctypes.data + 256) if kv.size else None, KV_ROW_BYTES,
                           idx, idx.shape[0],
                           swc.ctypes.data if swc.size else None,
                           sws.ctypes.data if sws.size else None, swc.shape[0],
                           float(softmax_scale), out, lse)
    return out, lse


# --------------------------------------------------------------------------
# causal visibility (prefill)
# --------------------------------------------------------------------------
TOKENS_PER_ENTRY = 4


def visible_entries(q_pos: Optional[int], n_entries: int) -> int:
    """Number of compressed entries a query may select.

    [B: CSA2：三层压缩一次吃满]: along the sequence every few tokens (4 in these workloads)
    become one compressed entry.  Reading: entry j summarises tokens 4j..4j+3 and exists for
    the query at absolute token position p only when all four are known, i.e. when
    4j + 3 <= p.  Decode (q_pos None): the query follows the whole context, so every entry
    is visible.  Written out as the definition: count the entries j < n_entries that pass.
    """
    if q_pos is None:
        return int(n_entries)
    j = np.arange(int(n_entries), dtype=np.int64)
    return int(np.count_nonzero(TOKENS_PER_ENTRY * j + (TOKENS_PER_ENTRY - 1) <= int(q_pos)))


# --------------------------------------------------------------------------
# sliding window
# --------------------------------------------------------------------------
SWA_WINDOW = 128


def window_tokens(q_pos: int, window: int = SWA_WINDOW) -> np.ndarray:
    """Absolute positions of the tokens in the sliding window of the query at position q_pos.

    [B: FP4 量化 + Bounded Replay]: the sliding window is cut down to the most recent 128
    tokens.  Reading: the query at token p sees token u through the window exactly when u is
    one of the `window` most recent tokens up to and including p, i.e. p - window < u <= p and
    u >= 0.  Written out as that definition over the candidate tokens 0..p, ascending.
    """
    p = int(q_pos)
    if p < 0:
        return np.zeros(0, np.int64)
    u = np.arange(p + 1, dtype=np.int64)
    return u[(u > p - int(window)) & (u <= p)]


# --------------------------------------------------------------------------
# layer group (mode table)
# --------------------------------------------------------------------------
FULL, REINDEX, REUSE = "F", "I", "U"


def layer_group_indices(modes: Sequence[str], layer_index_inputs, k_codes, k_scales,
                        n_vis: int, K: int, P: int):
    """Per-layer selected indices of one query row under a mode table.

    [B: CSA2：三层压缩一次吃满]: Full computes its own indexer query and runs the whole
    pipeline; Reindex reuses the earlier layer's keys and re-scores with its own query;
    Reuse takes the previous layer's top-K as is.  Reading: a Reindex layer searches
    the pool of the group's Full layer; Reuse copies the immediately preceding layer.

    layer_index_inputs[l] = (q_codes, q_scales, w) or None for Reuse layers.
    Returns a list of (idx, cnt).
    """
    out = []
    pool = pool_len = None
    need_pool = REINDEX in modes
    for l, m in enumerate(modes):
        if m == FULL:
            qc, qs, w = layer_index_inputs[l]
            idx, cnt, pool, pool_len, _ = full_index(qc, qs, w, k_codes, k_scales, n_vis, K,
                                                     P if need_pool else 0)
        elif m == REINDEX:
            if pool is None:
                raise ValueError("Reindex layer before any Full layer")
            qc, qs, w = layer_index_inputs[l]
            idx, cnt = reindex(qc, qs, w, k_codes, k_scales, pool, pool_len, K)
        elif m == REUSE:
            if not out:
                raise ValueError("Reuse layer before any Full layer")
            idx, cnt = out[-1]
        else:
            raise ValueError(f"unknown mode {m!r}")
        out.append((idx, cnt))
    return out


# --------------------------------------------------------------------------
# pool maintenance across decode steps
# --------------------------------------------------------------------------
def extend_pool(pool: np.ndarray, pool_len: int, n_ref: int, n_vis: int) -> np.ndarray:
    """Reindex candidates between pool refreshes: the kept pool (built when the sequence had
    n_ref entries) followed by every entry written since that the query may see (ids n_ref ..
    n_vis - 1), ascending."""
    kept = np.asarray(pool[:pool_len], np.int32)
    new = np.arange(int(n_ref), max(int(n_ref), int(n_vis)), dtype=np.int32)
    return np.concatenate([kept, new]).astype(np.int32)


def decode_steps_with_pool(modes: Sequence[str], step_inputs, k_codes, k_scales, n_steps: Sequence[int],
                           K: int, P: int, R: int):
    """Per-step, per-layer selections of one query row over consecutive decode steps, with the
    candidate pool kept across steps.

    [A: 压缩吸收注意力（二代）]: the first layer's scan picks a candidate pool that the later layers
    search.  The pages do not say how a pool is kept or refreshed as the context grows; the rule
    here (this library's own, documented with the layer group) is:
      * at steps s with s % R == 0 the Full layer's scan rebuilds the pool -- the top-min(P, n)
        of its own order, as in layer_group_indices -- and records n_ref = n, the entry count;
      * at the other steps the pool is kept, and the Reindex layers search the kept pool followed
        by every entry written since the rebuild (ids n_ref .. n - 1);
      * the Full layer's own top-K is always taken over the whole visible context.
    R = 1 rebuilds the pool every step, which is layer_group_indices step by step.

    step_inputs[s][l] = (q_codes, q_scales, w) or None (Reuse); n_steps[s] = visible entries at
    step s (non-decreasing).  Returns [step][layer] -> (idx, cnt).
    """
    out = []
    pool = pool_len = None
    n_ref = 0
    for s, n in enumerate(n_steps):
        refresh = (s % R) == 0 or pool is None
        res = []
        cand = None
        for l, m in enumerate(modes):
            if m == FULL:
                qc, qs, w = step_inputs[s][l]
                idx, cnt, p, pl, _ = full_index(qc, qs, w, k_codes, k_scales, n, K, P if refresh else 0)
                if refresh:
                    pool, pool_len, n_ref = p, pl, int(n)
                cand = pool[:pool_len] if refresh else extend_pool(pool, pool_len, n_ref, n)
            elif m == REINDEX:
                if cand is None:
                    raise ValueError("Reindex layer before any Full layer")
                qc, qs, w = step_inputs[s][l]
                idx, cnt = reindex(qc, qs, w, k_codes, k_scales, cand, len(cand), K)
            elif m == REUSE:
                if not res:
                    raise ValueError("Reuse layer before any Full layer")
                idx, cnt = res[-1]
            else:
                raise ValueError(f"unknown mode {m!r}")
            res.append((idx, cnt))
        out.append(res)
    return out
