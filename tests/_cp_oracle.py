"""Oracle-side shard of a context-parallel decode (tests only).

Same interface as compressed_sparse_attention_quantize_b200.context_parallel.DeviceShard, on CPU
tensors: every step is the oracle's own index scoring, top-K and fp64 attention restricted to the
shard, so the decomposition and the exchanges can be checked with gloo ranks on the CPU.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from compressed_sparse_attention_quantize_b200 import synth


def shard_bounds(n: int, g: int, G: int):
    return (n * g) // G, (n * (g + 1)) // G


class OracleShard:
    """Shard g of G of every sequence of `wl` (T = 1 decode rows)."""

    def __init__(self, wl: synth.Workload, seqs, g: int, G: int, softmax_scale: float):
        self.wl, self.seqs, self.g, self.G = wl, seqs, g, G
        self.softmax_scale = softmax_scale
        self.K = wl.K
        self.rows = wl.B * wl.T
        self.lo = np.array([shard_bounds(wl.n_entries[b], g, G)[0] for b in range(wl.B)], np.int64)
        self.hi = np.array([shard_bounds(wl.n_entries[b], g, G)[1] for b in range(wl.B)], np.int64)
        self.shard_lo = torch.from_numpy(self.lo.copy())
        self.owns_window = g == G - 1

    def local_topk(self, l: int):
        K, rows = self.K, self.rows
        scores = np.full((rows, K), -np.inf, np.float32)
        ids = np.full((rows, K), -1, np.int32)
        cnt = np.zeros((rows,), np.int32)
        for r in range(rows):
            b = r // self.wl.T
            os_ = self.seqs[b]
            L = os_.layer(l)
            lo, hi = int(self.lo[b]), int(self.hi[b])
            s = oracle.index_scores(L["qc"][0], L["qs"][0], L["w"][0], os_.k_codes[lo:hi], os_.k_scales[lo:hi])
            idx, c = oracle.topk(s, K)
            ids[r] = idx
            cnt[r] = c
            scores[r, :c] = s[idx[:c]]
        return torch.from_numpy(scores), torch.from_numpy(ids), torch.from_numpy(cnt)

    def merge_topk(self, scores_g, ids_g, cnt_g, lo_g):
        K, rows = self.K, self.rows
        idx = np.full((rows, K), -1, np.int32)
        cnt = np.zeros((rows,), np.int32)
        for r in range(rows):
            b = r // self.wl.T
            sc, gid = [], []
            for g in range(scores_g.shape[0]):
                c = int(cnt_g[g, r])
                sc.append(scores_g[g, r, :c].numpy())
                gid.append(ids_g[g, r, :c].numpy().astype(np.int64) + int(lo_g[g, b]))
            sc = np.concatenate(sc).astype(np.float32)
            gid = np.concatenate(gid).astype(np.int32)
            idx[r], cnt[r] = oracle.topk(sc, K, ids=gid)
        return torch.from_numpy(idx), torch.from_numpy(cnt)

    def attention(self, l: int, idx, cnt):
        H = self.wl.H
        rows = self.rows
        out = np.zeros((rows, H, 512), np.float64)
        lse = np.zeros((rows, H), np.float64)
        for r in range(rows):
            b = r // self.wl.T
            os_ = self.seqs[b]
            L = os_.layer(l)
            lo, hi = int(self.lo[b]), int(self.hi[b])
            sel = idx[r].numpy()
            mine = np.where((sel >= lo) & (sel < hi), sel - lo, -1).astype(np.int32)
            st, ln = synth.swa_window(self.wl, b)
            s0, n = int(st[0]), int(ln[0]) if self.owns_window else 0
            out[r], lse[r] = oracle.attention(L["q"][0], os_.kv_rows[lo:hi], mine, L["swc"][s0:s0 + n],
                                              L["sws"][s0:s0 + n], self.softmax_scale)
        return torch.from_numpy(out), torch.from_numpy(lse)

    @staticmethod
    def merge_attention(outs_g, lses_g):
        lses = lses_g.numpy()
        outs = outs_g.numpy()
        M = lses.max(axis=0)
        w = np.where(np.isfinite(lses), np.exp(lses - np.where(np.isfinite(M), M, 0.0)), 0.0)
        L = w.sum(axis=0)
        out = (w[..., None] * outs).sum(axis=0) / np.where(L > 0, L, 1.0)[..., None]
        lse = np.where(L > 0, M + np.log(np.where(L > 0, L, 1.0)), -np.inf)
        return out, lse
