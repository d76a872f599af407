"""CSA2 (Compressed Sparse Attention 2) hot path for NVIDIA B200 -- Python binding.

A thin ctypes layer over ``libcsa2.so`` (the C ABI declared in ``include/csa2.h``).
It only marshals arguments: every step runs in the library's CUDA kernels.  PyTorch
tensors are accepted wherever the C call takes a device pointer; the current
PyTorch CUDA stream is used unless ``stream`` is given.

There is no CPU fallback: if the library is missing or no CUDA device is present,
calls raise ``CSA2Error``.  Build with ``python -m compressed_sparse_attention_quantize_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

__all__ = [
    "CSA2Error", "lib", "library_path",
    "csa2_quantize_kv", "csa2_quantize_kv_batch", "quant_job", "QuantJob", "csa2_compress_quantize_kv", "csa2_index_topk", "csa2_index_topk_workspace_size",
    "csa2_index_topk_scored", "csa2_topk_merge_shards", "csa2_topk_merge_shards_workspace_size",
    "csa2_attn_merge_shards", "csa2_sparse_attn_shard", "csa2_pool_extend",
    "csa2_sparse_attn", "csa2_sparse_attn_workspace_size", "csa2_sparse_attn_plan", "csa2_sparse_attn_noalloc",
    "csa2_layer_group", "csa2_layer_group_workspace_size", "csa2_device_error", "csa2_selftest_bounded_wait",
    "csa2_status_string", "csa2_version", "csa2_launch_count", "GroupDesc", "LayerDesc",
    "csa2_host_alloc", "csa2_host_free", "host_empty",
    "FMT_FP4", "FMT_FP8_TOKEN", "DTYPE_F32", "DTYPE_BF16", "MODE_FULL", "MODE_REINDEX",
    "MODE_REUSE", "CSA2_OK", "CSA2_ERR_INVALID_ARG", "CSA2_ERR_SHAPE", "CSA2_ERR_TIMEOUT",
]

CSA2_OK = 0
CSA2_ERR_INVALID_ARG = 1
CSA2_ERR_SHAPE = 2
CSA2_ERR_TIMEOUT = 6

FMT_FP4 = 0
FMT_FP8_TOKEN = 1
DTYPE_F32 = 0
DTYPE_BF16 = 1
MODE_FULL = 0
MODE_REINDEX = 1
MODE_REUSE = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libcsa2.so")
_lib = None

_vp = ctypes.c_void_p
_i32 = ctypes.c_int
_i64 = ctypes.c_int64
_f32 = ctypes.c_float
_sz = ctypes.c_size_t


class CSA2Error(RuntimeError):
    pass


class QuantJob(ctypes.Structure):
    """Mirror of ``csa2_quant_job``."""
    _fields_ = [
        ("fmt", _i32), ("x_dtype", _i32), ("x", _vp), ("rows", _i64), ("dim", _i32), ("x_stride", _i64),
        ("codes", _vp), ("code_stride", _i64), ("scales", _vp), ("scale_stride", _i64), ("dst_rows", _vp),
    ]


# the csa2_version() the descriptors and signatures below mirror
ABI_VERSION = 6


class GroupDesc(ctypes.Structure):
    """Mirror of ``csa2_group_desc``."""
    _fields_ = [
        ("B", _i32), ("T", _i32), ("H", _i32), ("D", _i32), ("H_I", _i32), ("K", _i32), ("P", _i32),
        ("kv", _vp), ("kv_row_stride", _i64),
        ("k_codes", _vp), ("k_code_stride", _i64),
        ("k_scales", _vp), ("k_scale_stride", _i64),
        ("seq_start", _vp), ("n_entries", _vp), ("max_n", _i64),
        ("q_pos", _vp),
        ("swa_cap", _i32), ("swa_start", _vp), ("swa_len", _vp),
        ("softmax_scale", _f32), ("out_dtype", _i32),
        ("pool_keep", _vp), ("pool_keep_len", _vp), ("pool_keep_n", _vp), ("refresh", _i32), ("max_new", _i32),
    ]


class LayerDesc(ctypes.Structure):
    """Mirror of ``csa2_layer_desc``."""
    _fields_ = [
        ("mode", _i32), ("q", _vp), ("iq_codes", _vp), ("iq_scales", _vp), ("iw", _vp),
        ("swa_codes", _vp), ("swa_scale", _vp), ("out", _vp), ("lse", _vp), ("idx_out", _vp),
        ("ready_event", _vp), ("done_event", _vp), ("attn_ready_event", _vp),
    ]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libcsa2.so (raises CSA2Error when it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise CSA2Error(f"{_LIB_PATH} is missing; build it with "
                        "`python -m compressed_sparse_attention_quantize_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    L.csa2_status_string.restype = ctypes.c_char_p
    L.csa2_status_string.argtypes = [_i32]
    L.csa2_version.restype = _i32
    L.csa2_version.argtypes = []
    if L.csa2_version() != ABI_VERSION:
        raise CSA2Error(f"{_LIB_PATH} has ABI version {L.csa2_version()}, this binding expects "
                        f"{ABI_VERSION}; rebuild it with `python -m compressed_sparse_attention_quantize_b200.build`")
    L.csa2_host_alloc.restype = _i32
    L.csa2_host_alloc.argtypes = [_sz, ctypes.POINTER(_vp)]
    L.csa2_host_free.restype = _i32
    L.csa2_host_free.argtypes = [_vp]
    L.csa2_quantize_kv.restype = _i32
    L.csa2_quantize_kv.argtypes = [_i32, _vp, _i32, _i64, _i32, _i64, _vp, _i64, _vp, _i64, _vp, _vp]
    L.csa2_quantize_kv_batch.restype = _i32
    L.csa2_quantize_kv_batch.argtypes = [ctypes.POINTER(QuantJob), _i32, _vp]
    L.csa2_compress_quantize_kv.restype = _i32
    L.csa2_compress_quantize_kv.argtypes = [_vp, _i32, _i64, _i32, _i32, _i64, _vp, _i64, _vp, _i64,
                                            _vp, _i64, _vp, _vp]
    L.csa2_index_topk_scored.restype = _i32
    L.csa2_index_topk_scored.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _i64, _vp, _i64, _vp, _vp, _i64,
                                         _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp]
    L.csa2_topk_merge_shards_workspace_size.restype = _i32
    L.csa2_topk_merge_shards_workspace_size.argtypes = [_i32, _i32, _i32, ctypes.POINTER(_sz)]
    L.csa2_topk_merge_shards.restype = _i32
    L.csa2_topk_merge_shards.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp]
    L.csa2_sparse_attn_shard.restype = _i32
    L.csa2_sparse_attn_shard.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _i32,
                                         _vp, _vp, _i32, _vp, _vp, ctypes.c_float, _vp, _vp, _vp, _sz, _vp]
    L.csa2_attn_merge_shards.restype = _i32
    L.csa2_attn_merge_shards.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _i32, _vp, _vp]
    L.csa2_index_topk_workspace_size.restype = _i32
    L.csa2_index_topk_workspace_size.argtypes = [_i32, _i32, _i64, _i32, _i32, ctypes.POINTER(_sz)]
    L.csa2_index_topk.restype = _i32
    L.csa2_index_topk.argtypes = [_i32, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _i64, _vp, _i64,
                                  _vp, _vp, _i64, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _i32, _vp,
                                  _vp, _vp, _sz, _vp]
    L.csa2_pool_extend.restype = _i32
    L.csa2_pool_extend.argtypes = [_vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]
    L.csa2_sparse_attn_plan.restype = _i32
    L.csa2_sparse_attn_plan.argtypes = [_i32, _i32, _i32, ctypes.POINTER(_i32), ctypes.POINTER(_i32),
                                        ctypes.POINTER(_i32)]
    L.csa2_sparse_attn_workspace_size.restype = _i32
    L.csa2_sparse_attn_workspace_size.argtypes = [_i32, _i32, _i32, ctypes.POINTER(_sz)]
    L.csa2_sparse_attn.restype = _i32
    L.csa2_sparse_attn.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp, _vp, _i32,
                                   _vp, _vp, _i32, _vp, _vp, _f32, _vp, _i32, _vp, _vp, _sz, _vp]
    L.csa2_sparse_attn_noalloc.restype = _i32
    L.csa2_sparse_attn_noalloc.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp, _vp, _i32,
                                           _vp, _vp, _i32, _vp, _vp, _f32, _vp, _i32, _vp, _vp]
    L.csa2_layer_group_workspace_size.restype = _i32
    L.csa2_layer_group_workspace_size.argtypes = [ctypes.POINTER(GroupDesc), ctypes.POINTER(LayerDesc),
                                                  _i32, ctypes.POINTER(_sz)]
    L.csa2_layer_group.restype = _i32
    L.csa2_layer_group.argtypes = [ctypes.POINTER(GroupDesc), ctypes.POINTER(LayerDesc), _i32, _vp,
                                   _sz, _vp]
    L.csa2_device_error.restype = _i32
    L.csa2_device_error.argtypes = [_vp]
    L.csa2_selftest_bounded_wait.restype = _i32
    L.csa2_selftest_bounded_wait.argtypes = [_i32, _vp]
    L.csa2_last_error_string.restype = ctypes.c_char_p
    L.csa2_last_error_string.argtypes = []
    L.csa2_launch_count.restype = ctypes.c_uint64
    L.csa2_launch_count.argtypes = []
    _lib = L
    return L


def _ptr(x) -> Optional[int]:
    """Device address of a tensor (or an int address, or None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not getattr(x, "is_cuda", False):
        raise CSA2Error("expected a CUDA tensor or a device address")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        if not torch.cuda.is_available():
            raise CSA2Error("no CUDA device")
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int) -> None:
    if status != 0:
        msg = csa2_status_string(status)
        if status == 5:
            msg += " (" + lib().csa2_last_error_string().decode() + ")"
        raise CSA2Error(msg)


def csa2_status_string(status: int) -> str:
    return lib().csa2_status_string(int(status)).decode()


def csa2_version() -> int:
    return lib().csa2_version()


def csa2_quantize_kv(fmt, x, x_dtype, rows, dim, x_stride, codes, code_stride, scales, scale_stride,
                     dst_rows=None, stream=None) -> None:
    _check(lib().csa2_quantize_kv(fmt, _ptr(x), x_dtype, rows, dim, x_stride, _ptr(codes), code_stride,
                                  _ptr(scales), scale_stride, _ptr(dst_rows), _stream(stream)))


def quant_job(fmt, x, x_dtype, rows, dim, x_stride, codes, code_stride, scales, scale_stride,
              dst_rows=None) -> QuantJob:
    """One job of csa2_quantize_kv_batch (the arguments of csa2_quantize_kv)."""
    j = QuantJob()
    j.fmt, j.x_dtype, j.x, j.rows, j.dim, j.x_stride = fmt, x_dtype, _ptr(x), rows, dim, x_stride
    j.codes, j.code_stride, j.scales, j.scale_stride = _ptr(codes), code_stride, _ptr(scales), scale_stride
    j.dst_rows = _ptr(dst_rows)
    return j


def csa2_quantize_kv_batch(jobs: Sequence[QuantJob], stream=None) -> None:
    arr = (QuantJob * max(len(jobs), 1))(*jobs)
    _check(lib().csa2_quantize_kv_batch(arr, len(jobs), _stream(stream)))


def csa2_compress_quantize_kv(x, x_dtype, entries, ratio, dim, x_stride, w, w_stride, codes,
                              code_stride, scales, scale_stride, dst_rows=None, stream=None) -> None:
    _check(lib().csa2_compress_quantize_kv(_ptr(x), x_dtype, entries, ratio, dim, x_stride, _ptr(w),
                                           w_stride, _ptr(codes), code_stride, _ptr(scales),
                                           scale_stride, _ptr(dst_rows), _stream(stream)))


def csa2_index_topk_scored(q_codes, q_scales, w, B, T, H_I, k_codes, k_code_stride, k_scales,
                           k_scale_stride, seq_start, n_entries, max_n, q_pos, K, out_idx, out_cnt,
                           out_scores, workspace, ws_bytes, stream=None) -> None:
    _check(lib().csa2_index_topk_scored(_ptr(q_codes), _ptr(q_scales), _ptr(w), B, T, H_I, _ptr(k_codes),
                                        k_code_stride, _ptr(k_scales), k_scale_stride, _ptr(seq_start),
                                        _ptr(n_entries), max_n, _ptr(q_pos), K, _ptr(out_idx), _ptr(out_cnt),
                                        _ptr(out_scores), _ptr(workspace), ws_bytes, _stream(stream)))


def csa2_topk_merge_shards_workspace_size(G, rows, K_in) -> int:
    out = _sz(0)
    _check(lib().csa2_topk_merge_shards_workspace_size(G, rows, K_in, ctypes.byref(out)))
    return out.value


def csa2_topk_merge_shards(scores, ids, id_offset, cnt, G, rows, K_in, K, out_idx, out_cnt, workspace,
                           ws_bytes, stream=None) -> None:
    _check(lib().csa2_topk_merge_shards(_ptr(scores), _ptr(ids), _ptr(id_offset), _ptr(cnt), G, rows, K_in, K,
                                        _ptr(out_idx), _ptr(out_cnt), _ptr(workspace), ws_bytes,
                                        _stream(stream)))


def csa2_sparse_attn_shard(q, B, T, H, D, kv, kv_row_stride, seq_start, shard_lo, shard_n, idx, cnt, K,
                           swa_codes, swa_scale, swa_cap, swa_start, swa_len, softmax_scale, out, lse,
                           workspace, ws_bytes, stream=None) -> None:
    _check(lib().csa2_sparse_attn_shard(_ptr(q), B, T, H, D, _ptr(kv), kv_row_stride, _ptr(seq_start),
                                        _ptr(shard_lo), _ptr(shard_n), _ptr(idx), _ptr(cnt), K, _ptr(swa_codes),
                                        _ptr(swa_scale), swa_cap, _ptr(swa_start), _ptr(swa_len),
                                        ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                        ws_bytes, _stream(stream)))


def csa2_attn_merge_shards(outs, lses, G, rows, H, D, out, out_dtype, lse=None, stream=None) -> None:
    _check(lib().csa2_attn_merge_shards(_ptr(outs), _ptr(lses), G, rows, H, D, _ptr(out), out_dtype, _ptr(lse),
                                        _stream(stream)))


def csa2_index_topk_workspace_size(mode, rows, max_n, K, P) -> int:
    out = _sz(0)
    _check(lib().csa2_index_topk_workspace_size(mode, rows, max_n, K, P, ctypes.byref(out)))
    return out.value


def csa2_index_topk(mode, q_codes, q_scales, w, B, T, H_I, k_codes, k_code_stride, k_scales,
                    k_scale_stride, seq_start, n_entries, max_n, q_pos, pool, pool_len, P_in, K,
                    out_idx, out_cnt, P, out_pool, out_pool_len, workspace, ws_bytes,
                    stream=None) -> None:
    _check(lib().csa2_index_topk(mode, _ptr(q_codes), _ptr(q_scales), _ptr(w), B, T, H_I,
                                 _ptr(k_codes), k_code_stride, _ptr(k_scales), k_scale_stride,
                                 _ptr(seq_start), _ptr(n_entries), max_n, _ptr(q_pos), _ptr(pool),
                                 _ptr(pool_len), P_in, K, _ptr(out_idx), _ptr(out_cnt), P,
                                 _ptr(out_pool), _ptr(out_pool_len), _ptr(workspace), ws_bytes,
                                 _stream(stream)))


def csa2_host_alloc(nbytes: int) -> int:
    """Page-locked host buffer of at least ``nbytes`` on 2 MB pages (address as an int)."""
    p = _vp()
    _check(lib().csa2_host_alloc(int(nbytes), ctypes.byref(p)))
    return int(p.value)


def csa2_host_free(ptr: int) -> None:
    _check(lib().csa2_host_free(ptr))


def host_empty(shape, dtype):
    """A CPU torch tensor in a csa2_host_alloc buffer (page-locked, 2 MB pages, zero-filled by
    the calling thread); the buffer is freed when the tensor and its views are gone.  Use it for
    the inputs and outputs a step copies between host and device."""
    import weakref

    import numpy as np
    import torch
    shape = tuple(int(d) for d in shape)
    numel = 1
    for d in shape:
        numel *= d
    if numel == 0:
        return torch.empty(shape, dtype=dtype)
    nbytes = numel * torch.empty((), dtype=dtype).element_size()
    ptr = csa2_host_alloc(nbytes)
    buf = (ctypes.c_uint8 * nbytes).from_address(ptr)
    weakref.finalize(buf, lib().csa2_host_free, ptr)
    raw = torch.from_numpy(np.frombuffer(buf, dtype=np.uint8))   # holds buf through numpy
    return raw.view(dtype)[:numel].view(shape)


def csa2_pool_extend(pool, pool_len, P_in, n_ref, n_entries, q_pos, B, T, P_out, out_pool, out_len,
                     stream=None) -> None:
    _check(lib().csa2_pool_extend(_ptr(pool), _ptr(pool_len), P_in, _ptr(n_ref), _ptr(n_entries), _ptr(q_pos),
                                  B, T, P_out, _ptr(out_pool), _ptr(out_len), _stream(stream)))


def csa2_sparse_attn_plan(rows, H, K):
    """(hgroups, splits, keys_per_split) of a csa2_sparse_attn launch on the current device."""
    hg, sp, kps = _i32(0), _i32(0), _i32(0)
    _check(lib().csa2_sparse_attn_plan(rows, H, K, ctypes.byref(hg), ctypes.byref(sp), ctypes.byref(kps)))
    return hg.value, sp.value, kps.value


def csa2_sparse_attn_workspace_size(rows, H, K) -> int:
    out = _sz(0)
    _check(lib().csa2_sparse_attn_workspace_size(rows, H, K, ctypes.byref(out)))
    return out.value


def csa2_sparse_attn(q, B, T, H, D, kv, kv_row_stride, seq_start, n_entries, idx, cnt, K, swa_codes,
                     swa_scale, swa_cap, swa_start, swa_len, softmax_scale, out, out_dtype, lse, workspace,
                     ws_bytes, stream=None) -> None:
    _check(lib().csa2_sparse_attn(_ptr(q), B, T, H, D, _ptr(kv), kv_row_stride, _ptr(seq_start),
                                  _ptr(n_entries), _ptr(idx), _ptr(cnt), K, _ptr(swa_codes), _ptr(swa_scale), swa_cap,
                                  _ptr(swa_start), _ptr(swa_len), float(softmax_scale), _ptr(out),
                                  out_dtype, _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)))


def csa2_sparse_attn_noalloc(q, B, T, H, D, kv, kv_row_stride, seq_start, n_entries, idx, cnt, K,
                             swa_codes, swa_scale, swa_cap, swa_start, swa_len, softmax_scale, out,
                             out_dtype, lse, stream=None) -> None:
    """csa2_sparse_attn without a workspace argument, for callers that cannot allocate device
    memory: the scratch lives in a fixed array inside the library (see include/csa2.h)."""
    _check(lib().csa2_sparse_attn_noalloc(_ptr(q), B, T, H, D, _ptr(kv), kv_row_stride, _ptr(seq_start),
                                          _ptr(n_entries), _ptr(idx), _ptr(cnt), K, _ptr(swa_codes), _ptr(swa_scale),
                                          swa_cap, _ptr(swa_start), _ptr(swa_len), float(softmax_scale),
                                          _ptr(out), out_dtype, _ptr(lse), _stream(stream)))


def _layers_array(layers: Sequence[LayerDesc]):
    arr = (LayerDesc * len(layers))(*layers)
    return arr


def csa2_layer_group_workspace_size(g: GroupDesc, layers: Sequence[LayerDesc]) -> int:
    out = _sz(0)
    arr = _layers_array(layers)
    _check(lib().csa2_layer_group_workspace_size(ctypes.byref(g), arr, len(layers), ctypes.byref(out)))
    return out.value


def csa2_layer_group(g: GroupDesc, layers: Sequence[LayerDesc], workspace, ws_bytes,
                     stream=None) -> None:
    arr = _layers_array(layers)
    _check(lib().csa2_layer_group(ctypes.byref(g), arr, len(layers), _ptr(workspace), ws_bytes,
                                  _stream(stream)))


def csa2_device_error(stream=None) -> int:
    return lib().csa2_device_error(_stream(stream))


def csa2_selftest_bounded_wait(skip_arrival: bool, stream=None) -> None:
    """Launch the bounded-wait self-test; with skip_arrival the next csa2_device_error
    returns CSA2_ERR_TIMEOUT (6)."""
    _check(lib().csa2_selftest_bounded_wait(1 if skip_arrival else 0, _stream(stream)))


def csa2_launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(lib().csa2_launch_count())
