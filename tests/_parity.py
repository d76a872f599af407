"""Helpers for CUDA-vs-oracle parity tests (tests only).

The oracle regenerates the same seeded inputs (compressed_sparse_attention_quantize_b200.synth),
quantises them with its own code and computes the reference for chosen query rows.
"""
from __future__ import annotations

import math
from functools import lru_cache

import numpy as np

import oracle
from compressed_sparse_attention_quantize_b200 import synth

# Attention tolerance (stated with the workload): relative L2 <= 1e-3 and
# max-abs error <= 2e-3 * RMS(reference output), per query row.
REL_L2 = 1e-3
MAX_ABS_VS_RMS = 2e-3


class OracleSeq:
    """Oracle-side quantised caches of one sequence."""

    def __init__(self, wl: synth.Workload, b: int):
        self.wl, self.b = wl, b
        kc, ks = oracle.quantize_fp4(synth.kv_latent(wl, b))
        self.kv_rows = oracle.pack_kv_rows(kc, ks)
        self.k_codes, self.k_scales = oracle.quantize_fp4(synth.index_keys(wl, b))
        self._layer = {}

    def layer(self, l: int):
        if l not in self._layer:
            wl, b = self.wl, self.b
            iq = synth.index_query(wl, l, b).reshape(wl.T * wl.HI, 64)
            qc, qs = oracle.quantize_fp4(iq)
            w = synth.head_weights(wl, l, b)
            swc, sws = oracle.quantize_fp8_token(synth.swa_latent(wl, l, b))
            q = synth.main_query_bf16(wl, l, b)
            self._layer[l] = dict(qc=qc.reshape(wl.T, wl.HI, 32), qs=qs.reshape(wl.T, wl.HI, 4), w=w,
                                  swc=swc, sws=sws, q=q)
        return self._layer[l]

    def indices(self, t: int, modes):
        wl = self.wl
        inputs = []
        for l, m in enumerate(modes):
            if m == "U":
                inputs.append(None)
            else:
                L = self.layer(l)
                inputs.append((L["qc"][t], L["qs"][t], L["w"][t]))
        qp = None if wl.prefill_start is None else int(wl.q_pos(self.b)[t])
        n_vis = oracle.visible_entries(qp, wl.n_entries[self.b])
        return oracle.layer_group_indices(modes, inputs, self.k_codes, self.k_scales, n_vis, wl.K,
                                          wl.P)

    def window_slots(self, t: int):
        """Window-buffer slots of the tokens the oracle puts in query t's window."""
        qp = int(self.wl.q_pos(self.b)[t])
        return np.array([synth.window_slot(self.wl, self.b, u) for u in oracle.window_tokens(qp)],
                        np.int64)

    def attention(self, l: int, t: int, idx, softmax_scale):
        L = self.layer(l)
        slots = self.window_slots(t)
        return oracle.attention(L["q"][t], self.kv_rows, idx, L["swc"][slots], L["sws"][slots],
                                softmax_scale)


def check_attention(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    err = got - ref
    l2 = float(np.linalg.norm(err)) / max(float(np.linalg.norm(ref)), 1e-300)
    mx = float(np.abs(err).max()) if err.size else 0.0
    assert l2 <= REL_L2, f"{what}: relative L2 {l2:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_VS_RMS * rms + 1e-30, f"{what}: max-abs {mx:.3e} > {MAX_ABS_VS_RMS}*rms({rms:.3e})"
    return l2, mx / rms if rms else 0.0


def near_tie_swaps(scores: np.ndarray, ref_idx: np.ndarray, got_idx: np.ndarray, rel: float = 1e-6):
    """Return (ok, n_swaps): selections that differ must sit within `rel` of the K-th score."""
    a = set(int(x) for x in ref_idx if x >= 0)
    b = set(int(x) for x in got_idx if x >= 0)
    diff = a ^ b
    if not diff:
        return True, 0
    kth = min(scores[list(a)]) if a else 0.0
    ok = all(abs(scores[j] - kth) <= rel * max(abs(kth), 1e-30) for j in diff)
    return ok, len(diff) // 2
