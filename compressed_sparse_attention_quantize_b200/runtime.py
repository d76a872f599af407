"""Device-side setup of a CSA2 workload and one call of the layer group.

``GroupRunner`` owns the caller-side buffers the C ABI expects (PyTorch allocates them):
the packed main-KV cache (288-byte rows), the indexer-key cache, and per layer the main
query, the quantised indexer query and head weights, the 8-bit window and the outputs.
All quantisation is done on the device with ``csa2_quantize_kv`` (quantise-on-write).
"""
from __future__ import annotations

import math
from typing import List, Optional

import numpy as np
import torch

from . import (DTYPE_BF16, DTYPE_F32, FMT_FP4, FMT_FP8_TOKEN, MODE_FULL, MODE_REINDEX, MODE_REUSE,
               GroupDesc, LayerDesc, csa2_layer_group, csa2_layer_group_workspace_size,
               csa2_quantize_kv, csa2_quantize_kv_batch, quant_job)
from . import synth

KV_ROW = 288
_MODE = {"F": MODE_FULL, "I": MODE_REINDEX, "U": MODE_REUSE}


def quantize_fp4_rows(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                      code_stride: int, scale_stride: int, dst_rows=None, stream=None):
    """Quantise float32/bf16 rows [rows, dim] into FP4 codes/scales (device buffers)."""
    rows, dim = x.shape
    dt = DTYPE_F32 if x.dtype == torch.float32 else DTYPE_BF16
    csa2_quantize_kv(FMT_FP4, x, dt, rows, dim, x.stride(0), codes, code_stride, scales,
                     scale_stride, dst_rows, stream)


def quantize_fp8_rows(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, dst_rows=None,
                      stream=None):
    rows, dim = x.shape
    dt = DTYPE_F32 if x.dtype == torch.float32 else DTYPE_BF16
    csa2_quantize_kv(FMT_FP8_TOKEN, x, dt, rows, dim, x.stride(0), codes, codes.stride(0), scales,
                     4, dst_rows, stream)


class GroupRunner:
    """Holds one workload on the device and runs its layer group through the C ABI."""

    def __init__(self, wl: synth.Workload, device="cuda", out_dtype=DTYPE_F32,
                 softmax_scale: Optional[float] = None, layers: Optional[int] = None):
        self.wl = wl
        self.dev = torch.device(device)
        self.out_dtype = out_dtype
        self.softmax_scale = (1.0 / math.sqrt(synth.D_LATENT)) if softmax_scale is None else softmax_scale
        modes = wl.modes if layers is None else wl.modes[:layers]
        self.modes = modes
        B, T, H, HI, K = wl.B, wl.T, wl.H, wl.HI, wl.K
        self.rows = B * T
        n = wl.n_entries
        starts = np.concatenate([[0], np.cumsum(n)[:-1]]).astype(np.int64)
        total = int(np.sum(n))
        self.total_entries = total
        self.max_n = int(max(n))
        d = self.dev
        self.seq_start = torch.from_numpy(starts).to(d)
        self.n_entries = torch.tensor(n, dtype=torch.int32, device=d)
        self.kv = torch.empty((max(total, 1), KV_ROW), dtype=torch.uint8, device=d)
        self.k_codes = torch.empty((max(total, 1), 32), dtype=torch.uint8, device=d)
        self.k_scales = torch.empty((max(total, 1), 4), dtype=torch.uint8, device=d)
        # caches: quantise-on-write, one sequence at a time (bounds host memory); the newest
        # entry of each sequence is kept in float for the per-step write (write_step)
        step_kv, step_ik, step_rows = [], [], []
        for b in range(B):
            s0 = int(starts[b])
            lat = torch.from_numpy(synth.kv_latent(wl, b)).to(d)
            quantize_fp4_rows(lat, self.kv[s0:], self.kv[s0:, 256:], KV_ROW, KV_ROW)
            if n[b] > 0:
                step_kv.append(lat[n[b] - 1:n[b]].clone())
                step_rows.append(s0 + n[b] - 1)
            del lat
            ik = torch.from_numpy(synth.index_keys(wl, b)).to(d)
            quantize_fp4_rows(ik, self.k_codes[s0:], self.k_scales[s0:], 32, 4)
            if n[b] > 0:
                step_ik.append(ik[n[b] - 1:n[b]].clone())
            del ik
        self.step_kv = torch.cat(step_kv) if step_kv else None
        self.step_ik = torch.cat(step_ik) if step_ik else None
        self.step_rows = torch.tensor(step_rows, dtype=torch.int64, device=d) if step_rows else None
        if step_rows:
            assert max(step_rows) < self.kv.shape[0] and min(step_rows) >= 0
        # query positions (prefill) and window slots
        if wl.prefill_start is not None:
            qp = np.concatenate([wl.q_pos(b) for b in range(B)]).astype(np.int32)
            self.q_pos = torch.from_numpy(qp).to(d)
        else:
            self.q_pos = None
        st, ln = zip(*[synth.swa_window(wl, b) for b in range(B)])
        self.swa_start = torch.from_numpy(np.concatenate(st).astype(np.int32)).to(d)
        self.swa_len = torch.from_numpy(np.concatenate(ln).astype(np.int32)).to(d)
        self.swa_cap = wl.swa_tokens()
        # every layer's window in one buffer (layer l holds rows l*B*swa_cap ..), so that one
        # scatter call writes all layers' window entries of a step
        win_rows = B * self.swa_cap
        self.swa_codes_all = torch.empty((len(modes) * win_rows, 512), dtype=torch.uint8, device=d)
        self.swa_scale_all = torch.empty((len(modes) * win_rows,), dtype=torch.float32, device=d)
        win_slots = self._step_window_slots()
        assert all(0 <= x < win_rows for x in win_slots)
        step_win_lat, step_win_rows = [], []
        # per layer
        self.layer_data = []
        odt = torch.float32 if out_dtype == DTYPE_F32 else torch.bfloat16
        for l, m in enumerate(modes):
            q = np.stack([synth.main_query_bf16(wl, l, b) for b in range(B)]).reshape(self.rows, H, 512)
            ld = {"q": torch.from_numpy(q.view(np.int16)).to(d)}
            if m != "U":
                iq = np.stack([synth.index_query(wl, l, b) for b in range(B)]).reshape(self.rows * HI, 64)
                iqt = torch.from_numpy(iq).to(d)
                ld["iq_codes"] = torch.empty((self.rows * HI, 32), dtype=torch.uint8, device=d)
                ld["iq_scales"] = torch.empty((self.rows * HI, 4), dtype=torch.uint8, device=d)
                quantize_fp4_rows(iqt, ld["iq_codes"], ld["iq_scales"], 32, 4)
                ld["iq_f32"] = iqt
                w = np.stack([synth.head_weights(wl, l, b) for b in range(B)]).reshape(self.rows, HI)
                ld["iw"] = torch.from_numpy(np.ascontiguousarray(w)).to(d)
            sw = np.stack([synth.swa_latent(wl, l, b) for b in range(B)]).reshape(B * self.swa_cap, 512)
            swt = torch.from_numpy(sw).to(d)
            ld["swa_codes"] = self.swa_codes_all[l * win_rows:(l + 1) * win_rows]
            ld["swa_scale"] = self.swa_scale_all[l * win_rows:(l + 1) * win_rows]
            quantize_fp8_rows(swt, ld["swa_codes"], ld["swa_scale"])
            # the window entries of this step's tokens, for the per-step write
            if win_slots:
                step_win_lat.append(swt.index_select(0, torch.tensor(win_slots, dtype=torch.int64, device=d)))
                step_win_rows.extend(l * win_rows + x for x in win_slots)
            del swt
            ld["out"] = torch.empty((self.rows, H, 512), dtype=odt, device=d)
            ld["lse"] = torch.empty((self.rows, H), dtype=torch.float32, device=d)
            ld["idx"] = torch.empty((self.rows, K), dtype=torch.int32, device=d)
            self.layer_data.append(ld)
        self.step_win_lat = torch.cat(step_win_lat).contiguous() if step_win_lat else None
        self.step_win_rows = (torch.tensor(step_win_rows, dtype=torch.int64, device=d)
                              if step_win_rows else None)
        if step_win_rows:
            assert max(step_win_rows) < self.swa_codes_all.shape[0]
        self.entry_jobs, self.window_jobs, self.query_jobs = self._write_jobs()
        self.g = self._group_desc()
        self.layer_descs = [self._layer_desc(l) for l in range(len(modes))]
        self.ws_bytes = csa2_layer_group_workspace_size(self.g, self.layer_descs)
        self.workspace = torch.empty((self.ws_bytes,), dtype=torch.uint8, device=d)
        torch.cuda.synchronize()

    def _step_window_slots(self) -> List[int]:
        """Rows b * swa_cap + slot of the window entries this step's tokens write.  Decode: the
        128-slot ring holds token p in slot p % 128, so the current token is slot (ctx - 1) % 128
        (none for an empty context).  Prefill: the buffer holds the 127 tokens before the chunk
        and then the chunk, so chunk token t is slot 127 + t."""
        wl = self.wl
        out = []
        for b in range(wl.B):
            if wl.prefill_start is None:
                if wl.ctx_tokens[b] > 0:
                    out.append(b * self.swa_cap + (wl.ctx_tokens[b] - 1) % synth.SWA_WINDOW)
            else:
                out.extend(b * self.swa_cap + (synth.SWA_WINDOW - 1) + t for t in range(wl.T))
        return out

    def _write_jobs(self, kv=None, ik=None, win=None, iq=None):
        """csa2_quantize_kv_batch jobs of a step's writes: (entry jobs, window jobs, query jobs),
        from the runner's device inputs or from the given device tensors of the same shapes (kv,
        ik: the new entries' latents and indexer keys; win: the window tokens; iq: a list with
        each Full/Reindex layer's indexer query, None elsewhere)."""
        def fp4(x, codes, scales, cs, ss, dst=None):
            dt = DTYPE_F32 if x.dtype == torch.float32 else DTYPE_BF16
            return quant_job(FMT_FP4, x, dt, x.shape[0], x.shape[1], x.stride(0), codes, cs, scales, ss, dst)
        kv = self.step_kv if kv is None else kv
        ik = self.step_ik if ik is None else ik
        win = self.step_win_lat if win is None else win
        entries, windows, queries = [], [], []
        if self.step_rows is not None:
            entries.append(fp4(kv, self.kv, self.kv[:, 256:], KV_ROW, KV_ROW, self.step_rows))
            entries.append(fp4(ik, self.k_codes, self.k_scales, 32, 4, self.step_rows))
        if self.step_win_rows is not None:
            windows.append(quant_job(FMT_FP8_TOKEN, win, DTYPE_F32, win.shape[0], win.shape[1], win.stride(0),
                                     self.swa_codes_all, self.swa_codes_all.stride(0), self.swa_scale_all, 4,
                                     self.step_win_rows))
        for l, ld in enumerate(self.layer_data):
            if "iq_f32" in ld:
                x = ld["iq_f32"] if iq is None or iq[l] is None else iq[l]
                queries.append(fp4(x, ld["iq_codes"], ld["iq_scales"], 32, 4))
        return entries, windows, queries

    def write_jobs(self, kv=None, ik=None, win=None, iq=None):
        """The step's quantise-on-write jobs (entries, windows, queries) reading the given device
        tensors instead of the runner's own inputs (see _write_jobs)."""
        return self._write_jobs(kv, ik, win, iq)

    def _group_desc(self) -> GroupDesc:
        wl = self.wl
        g = GroupDesc()
        g.B, g.T, g.H, g.D, g.H_I, g.K, g.P = wl.B, wl.T, wl.H, 512, wl.HI, wl.K, wl.P
        g.kv, g.kv_row_stride = self.kv.data_ptr(), KV_ROW
        g.k_codes, g.k_code_stride = self.k_codes.data_ptr(), 32
        g.k_scales, g.k_scale_stride = self.k_scales.data_ptr(), 4
        g.seq_start, g.n_entries, g.max_n = self.seq_start.data_ptr(), self.n_entries.data_ptr(), self.max_n
        g.q_pos = self.q_pos.data_ptr() if self.q_pos is not None else None
        g.swa_cap, g.swa_start, g.swa_len = self.swa_cap, self.swa_start.data_ptr(), self.swa_len.data_ptr()
        g.softmax_scale, g.out_dtype = self.softmax_scale, self.out_dtype
        return g

    def keep_pool(self, max_new: int) -> None:
        """Keep the Reindex layers' candidate pool across decode calls (csa2_group_desc's
        pool_keep): ``run(refresh=True)`` rebuilds it, ``run(refresh=False)`` searches it followed
        by the at most ``max_new`` entries per sequence written since.  The first call after
        this one must refresh."""
        d, wl = self.dev, self.wl
        self.pool_keep = torch.full((self.rows, max(wl.P, 1)), -1, dtype=torch.int32, device=d)
        self.pool_keep_len = torch.zeros((self.rows,), dtype=torch.int32, device=d)
        self.pool_keep_n = torch.zeros((wl.B,), dtype=torch.int32, device=d)
        g = self.g
        g.pool_keep, g.pool_keep_len = self.pool_keep.data_ptr(), self.pool_keep_len.data_ptr()
        g.pool_keep_n, g.max_new, g.refresh = self.pool_keep_n.data_ptr(), int(max_new), 1
        self.ws_bytes = csa2_layer_group_workspace_size(self.g, self.layer_descs)
        self.workspace = torch.empty((self.ws_bytes,), dtype=torch.uint8, device=d)

    def _layer_desc(self, l: int) -> LayerDesc:
        ld = self.layer_data[l]
        L = LayerDesc()
        L.mode = _MODE[self.modes[l]]
        L.q = ld["q"].data_ptr()
        if "iq_codes" in ld:
            L.iq_codes, L.iq_scales, L.iw = ld["iq_codes"].data_ptr(), ld["iq_scales"].data_ptr(), ld["iw"].data_ptr()
        L.swa_codes, L.swa_scale = ld["swa_codes"].data_ptr(), ld["swa_scale"].data_ptr()
        L.out, L.lse, L.idx_out = ld["out"].data_ptr(), ld["lse"].data_ptr(), ld["idx"].data_ptr()
        return L

    def set_layer_events(self, ready=None, done=None, attn_ready=None) -> None:
        """Per-layer cudaEvent_t handles (ints, or None) that the group call waits on before a
        layer (``ready``) and before its attention (``attn_ready``), and records after it
        (``done``); see csa2_layer_group."""
        for l, L in enumerate(self.layer_descs):
            L.ready_event = ready[l] if ready else None
            L.done_event = done[l] if done else None
            L.attn_ready_event = attn_ready[l] if attn_ready else None

    def run(self, stream=None, refresh: Optional[bool] = None) -> None:
        """The layer group; ``refresh`` sets whether a kept pool (keep_pool) is rebuilt."""
        if refresh is not None:
            self.g.refresh = 1 if refresh else 0
        csa2_layer_group(self.g, self.layer_descs, self.workspace, self.ws_bytes, stream)

    def write_step(self, stream=None) -> None:
        """A decode step's quantise-on-write, from float inputs held on the device: the newest
        compressed entry of every sequence and its indexer key (FP4, written at its cache row),
        every Full/Reindex layer's indexer query (FP4), and every layer's window entries of the
        step's tokens (E4M3 + fp32 scale, at their window slots; one call for all layers).  The
        inputs are the ones the caches were built from, so the bytes written equal those already
        there and a step that runs write_step() then run() reads the same caches as run() alone.
        All of it is one csa2_quantize_kv_batch launch."""
        jobs = self.entry_jobs + self.window_jobs + self.query_jobs
        if jobs:
            csa2_quantize_kv_batch(jobs, stream)

    def write_entries(self, stream=None) -> None:
        """The newest compressed entry of every non-empty sequence (main KV, FP4) and its
        indexer key (FP4), each written at its cache row."""
        if self.step_rows is not None:
            quantize_fp4_rows(self.step_kv, self.kv, self.kv[:, 256:], KV_ROW, KV_ROW,
                              dst_rows=self.step_rows, stream=stream)
            quantize_fp4_rows(self.step_ik, self.k_codes, self.k_scales, 32, 4,
                              dst_rows=self.step_rows, stream=stream)

    def write_windows(self, stream=None) -> None:
        """Every layer's window entries of the step's tokens, in one scatter call."""
        if self.step_win_rows is not None:
            quantize_fp8_rows(self.step_win_lat, self.swa_codes_all, self.swa_scale_all,
                              dst_rows=self.step_win_rows, stream=stream)

    def write_queries(self, stream=None) -> None:
        """Every Full/Reindex layer's indexer query (FP4)."""
        for ld in self.layer_data:
            if "iq_f32" in ld:
                quantize_fp4_rows(ld["iq_f32"], ld["iq_codes"], ld["iq_scales"], 32, 4, stream=stream)

    def step(self, stream=None) -> None:
        """One whole decode step: the step's writes, then the layer group."""
        self.write_step(stream)
        self.run(stream)

    def capture(self, with_writes: bool = False) -> int:
        """Record one call of the layer group (preceded by the step's writes when
        ``with_writes``) into a CUDA graph, after a warm-up call so that the library's one-time
        attribute set-up happens outside the capture; ``replay()`` then launches it with one
        graph launch.  Returns the number of library kernels the graph holds.  The graph reads
        the current contents of the runner's buffers."""
        from . import csa2_launch_count
        fn = self.step if with_writes else self.run
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        n0 = csa2_launch_count()
        with torch.cuda.graph(graph):
            fn()
        self.graph = graph
        self.graph_kernels = csa2_launch_count() - n0
        return self.graph_kernels

    def replay(self) -> None:
        self.graph.replay()
