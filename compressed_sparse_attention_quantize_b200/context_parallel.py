"""Context-parallel decode: one long sequence's compressed entries split across GPUs.

[A] page "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径", section "压缩吸收注意力（二代）":
the indexer keeps the top 2048 blocks of the whole context (score descending, entry index
ascending on ties).  [B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型",
section "CSA2：三层压缩一次吃满": each layer attends once, with one joint softmax, over its
selection and its window.

Every GPU (rank g of G) holds a consecutive shard of each sequence's entries -- global entries
[lo_g[b], lo_g[b] + n_g[b]) -- in its own main-KV and indexer-key caches.  A decode layer is:

1. ``local_topk``: the shard's own Full-mode top-K with the scores of the chosen entries
   (``csa2_index_topk_scored``).
2. exchange: all-gather of the G scored lists.  The global top-K lies inside their union.
3. ``merge_topk``: the global top-K of the union (``csa2_topk_merge_shards``), the same set
   and order as one GPU scoring the whole sequence.
4. ``attention``: attention over the selected entries that live in this shard, plus the
   window on the rank that holds it (``csa2_sparse_attn_shard``): an fp32 output and its LSE.
5. exchange: all-gather of the G partial results.
6. ``merge_attention``: log-sum-exp merge (``csa2_attn_merge_shards``).

Reuse layers skip 1-3 and keep the previous selection.  The exchanges carry G x K (score, id)
pairs and G fp32 outputs per query row; every rank ends with the full result.  Ranks must call
``decode_layer`` in the same order (the collectives are matched by order).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import (DTYPE_F32, csa2_attn_merge_shards, csa2_index_topk_scored, csa2_index_topk_workspace_size,
               csa2_sparse_attn_shard, csa2_sparse_attn_workspace_size, csa2_topk_merge_shards,
               csa2_topk_merge_shards_workspace_size, MODE_FULL)


class Comm:
    """All-gather over the ranks that share the sequences (``torch.distributed``)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        """[G, *t.shape], rank order."""
        t = t.contiguous()
        parts = [torch.empty_like(t) for _ in range(self.size)]
        self.dist.all_gather(parts, t, group=self.group)
        return torch.stack(parts)


@dataclass
class LayerInputs:
    """One layer's per-rank inputs (device tensors).  iq_* / iw only for Full layers; the window
    tensors only matter on the rank that holds the window (others pass swa_len of zeros)."""
    q: torch.Tensor                 # bf16 bits (int16) [rows, H, D]
    swa_codes: torch.Tensor
    swa_scale: torch.Tensor
    swa_start: Optional[torch.Tensor]
    swa_len: torch.Tensor           # int32 [rows]
    iq_codes: Optional[torch.Tensor] = None
    iq_scales: Optional[torch.Tensor] = None
    iw: Optional[torch.Tensor] = None


class DeviceShard:
    """This GPU's shard of B sequences and the CUDA steps over it (through the C ABI)."""

    def __init__(self, kv, k_codes, k_scales, seq_start, shard_lo, shard_n, B, T, H, H_I, K, swa_cap,
                 softmax_scale, D=512):
        self.kv, self.k_codes, self.k_scales = kv, k_codes, k_scales
        self.seq_start, self.shard_lo, self.shard_n = seq_start, shard_lo, shard_n
        self.B, self.T, self.H, self.H_I, self.K, self.D = B, T, H, H_I, K, D
        self.swa_cap, self.softmax_scale = swa_cap, softmax_scale
        self.rows = B * T
        self.max_n = int(shard_n.max().item()) if B else 0
        dev = kv.device
        self.ws_idx = torch.empty(csa2_index_topk_workspace_size(MODE_FULL, self.rows, max(self.max_n, 1), K, 0),
                                  dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(csa2_sparse_attn_workspace_size(self.rows, H, K), dtype=torch.uint8, device=dev)

    def local_topk(self, li: LayerInputs):
        dev = self.kv.device
        ids = torch.empty((self.rows, self.K), dtype=torch.int32, device=dev)
        cnt = torch.empty((self.rows,), dtype=torch.int32, device=dev)
        scores = torch.empty((self.rows, self.K), dtype=torch.float32, device=dev)
        csa2_index_topk_scored(li.iq_codes, li.iq_scales, li.iw, self.B, self.T, self.H_I, self.k_codes, 32,
                               self.k_scales, 4, self.seq_start, self.shard_n, max(self.max_n, 1), None, self.K,
                               ids, cnt, scores, self.ws_idx, self.ws_idx.numel())
        return scores, ids, cnt

    def merge_topk(self, scores_g, ids_g, cnt_g, lo_g):
        """scores_g, ids_g: [G, rows, K]; cnt_g: [G, rows]; lo_g: [G, B] shard starts."""
        G = scores_g.shape[0]
        dev = scores_g.device
        offset = lo_g.to(torch.int64).repeat_interleave(self.T, dim=1).contiguous()       # [G, rows]
        ws = torch.empty(csa2_topk_merge_shards_workspace_size(G, self.rows, self.K), dtype=torch.uint8,
                         device=dev)
        idx = torch.empty((self.rows, self.K), dtype=torch.int32, device=dev)
        cnt = torch.empty((self.rows,), dtype=torch.int32, device=dev)
        csa2_topk_merge_shards(scores_g.contiguous(), ids_g.contiguous(), offset, cnt_g.contiguous(), G,
                               self.rows, self.K, self.K, idx, cnt, ws, ws.numel())
        return idx, cnt

    def attention(self, li: LayerInputs, idx, cnt):
        dev = self.kv.device
        out = torch.empty((self.rows, self.H, self.D), dtype=torch.float32, device=dev)
        lse = torch.empty((self.rows, self.H), dtype=torch.float32, device=dev)
        csa2_sparse_attn_shard(li.q, self.B, self.T, self.H, self.D, self.kv, 288, self.seq_start, self.shard_lo,
                               self.shard_n, idx, cnt, self.K, li.swa_codes, li.swa_scale, self.swa_cap,
                               li.swa_start, li.swa_len, self.softmax_scale, out, lse, self.ws_attn,
                               self.ws_attn.numel())
        return out, lse

    def merge_attention(self, outs_g, lses_g, out_dtype=DTYPE_F32):
        G = outs_g.shape[0]
        dt = torch.float32 if out_dtype == DTYPE_F32 else torch.bfloat16
        out = torch.empty((self.rows, self.H, self.D), dtype=dt, device=outs_g.device)
        lse = torch.empty((self.rows, self.H), dtype=torch.float32, device=outs_g.device)
        csa2_attn_merge_shards(outs_g.contiguous(), lses_g.contiguous(), G, self.rows, self.H, self.D, out,
                               out_dtype, lse)
        return out, lse


def decode_layer(comm, shard, li: LayerInputs, full: bool, prev=None, out_dtype=DTYPE_F32):
    """One layer on every rank: returns (idx, cnt, out, lse), identical on all ranks.
    `full`: run the indexer (Full layer); otherwise reuse `prev` = (idx, cnt)."""
    if full:
        scores, ids, cnt_local = shard.local_topk(li)
        scores_g = comm.all_gather(scores)
        ids_g = comm.all_gather(ids)
        cnt_g = comm.all_gather(cnt_local)
        lo_g = comm.all_gather(shard.shard_lo)
        idx, cnt = shard.merge_topk(scores_g, ids_g, cnt_g, lo_g)
    else:
        idx, cnt = prev
    out_l, lse_l = shard.attention(li, idx, cnt)
    outs_g = comm.all_gather(out_l)
    lses_g = comm.all_gather(lse_l)
    out, lse = shard.merge_attention(outs_g, lses_g, out_dtype)
    return idx, cnt, out, lse
