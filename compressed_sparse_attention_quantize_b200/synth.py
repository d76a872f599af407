"""Seeded synthetic inputs for the CSA2 hot path (shared by the tests, the bench and the oracle).

This module only draws random numbers in the shapes and distributions of the five
workloads; it holds none of the method's arithmetic (no quantisation, scoring,
selection or attention).  Every tensor is drawn from its own counter-keyed stream,
``numpy.random.default_rng(SeedSequence([seed, stream, layer, sequence]))``, so one
sequence of one layer can be regenerated alone (the full-size parity tests use that
to check sampled rows).

Distributions:
  * main-KV and sliding-window latents: N(0, 1), 512 wide, with 4 outlier channels
    (drawn without replacement once per workload) multiplied by 8;
  * main query: bf16 of N(0, 1/512);
  * indexer keys: N(0, 1), 64 wide; indexer queries: N(0, 1/64) per head;
  * indexer head weights: U(0, 1) float32.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

D_LATENT = 512
D_INDEX = 64
SWA_WINDOW = 128
TOKENS_PER_ENTRY = 4
OUTLIER_COUNT = 4
OUTLIER_GAIN = 8.0

# stream ids
_S_OUTLIER, _S_KV, _S_IDXK, _S_Q, _S_IQ, _S_W, _S_SWA, _S_LEN = 1, 2, 3, 4, 5, 6, 7, 8


@dataclass
class Workload:
    """Shape of one CSA2 workload (a group of layers over a batch of sequences)."""
    name: str
    seed: int
    B: int                      # sequences
    T: int                      # query tokens per sequence (1 = decode)
    n_entries: List[int]        # compressed entries per sequence (after this step's writes)
    H: int                      # main query heads
    HI: int                     # indexer heads
    K: int                      # top-K
    P: int                      # candidate-pool size (0 = no pool)
    modes: Tuple[str, ...]      # per layer: "F" Full, "I" Reindex, "U" Reuse
    ctx_tokens: List[int] = field(default_factory=list)   # context length per sequence (tokens)
    prefill_start: Optional[int] = None   # absolute position of the first query token (prefill)
    new_entries: int = 0        # entries written by this step (quantise-on-write), per sequence

    @property
    def layers(self) -> int:
        return len(self.modes)

    def q_pos(self, b: int) -> np.ndarray:
        """Absolute token position of each query of sequence b."""
        if self.prefill_start is None:
            return np.array([self.ctx_tokens[b] - 1], np.int64)
        return self.prefill_start + np.arange(self.T, dtype=np.int64)

    def swa_tokens(self) -> int:
        """Sliding-window slots held per sequence per layer."""
        if self.prefill_start is None:
            return SWA_WINDOW
        return self.T + SWA_WINDOW - 1


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed)] + [int(k) for k in key]))


def workload(i: int) -> Workload:
    """The five workloads: 0 tiny Full layer, 1 decode 128K, 2 Reindex 256K, 3 decode 1M,
    4 prefill chunk."""
    if i == 0:
        return Workload("tiny_full_4k", 0, B=1, T=1, n_entries=[1024], H=16, HI=4, K=64, P=0,
                        modes=("F",), ctx_tokens=[4096])
    if i == 1:
        return Workload("decode_128k_b32_F5U", 1, B=32, T=1, n_entries=[32768] * 32, H=64, HI=8,
                        K=2048, P=0, modes=("F", "U", "U", "U", "U", "U"), ctx_tokens=[131072] * 32)
    if i == 2:
        return Workload("reindex_256k_b16_FIUIUU", 2, B=16, T=1, n_entries=[65536] * 16, H=64, HI=8,
                        K=2048, P=16000, modes=("F", "I", "U", "I", "U", "U"),
                        ctx_tokens=[262144] * 16)
    if i == 3:
        rng = _rng(3, _S_LEN)
        ctx = rng.integers(512 * 1024, 1024 * 1024, size=4, endpoint=True)
        return Workload("decode_1m_b4_F5U", 3, B=4, T=1,
                        n_entries=[int(c) // TOKENS_PER_ENTRY for c in ctx], H=64, HI=8,
                        K=2048, P=0, modes=("F", "U", "U", "U", "U", "U"),
                        ctx_tokens=[int(c) for c in ctx])
    if i == 4:
        return Workload("prefill_4096_on_128k", 4, B=1, T=4096, n_entries=[32768 + 1024], H=64,
                        HI=8, K=2048, P=0, modes=("F",), ctx_tokens=[131072 + 4096],
                        prefill_start=131072, new_entries=1024)
    raise ValueError(i)


def scaled(wl: Workload, *, B=None, n=None, T=None, K=None, P=None, H=None, HI=None, modes=None,
           name=None) -> Workload:
    """A smaller copy of a workload with the same structure (for tests the oracle runs fully)."""
    B = wl.B if B is None else B
    n_entries = list(wl.n_entries[:B]) if n is None else ([n] * B if isinstance(n, int) else list(n))
    T = wl.T if T is None else T
    ctx = [x * TOKENS_PER_ENTRY for x in n_entries]
    pstart = None
    if wl.prefill_start is not None:
        pstart = ctx[0] - T
    return Workload(name or (wl.name + "_scaled"), wl.seed, B=B, T=T, n_entries=n_entries,
                    H=wl.H if H is None else H, HI=wl.HI if HI is None else HI,
                    K=wl.K if K is None else K, P=wl.P if P is None else P,
                    modes=wl.modes if modes is None else tuple(modes), ctx_tokens=ctx,
                    prefill_start=pstart, new_entries=(min(wl.new_entries, n_entries[0])
                                                       if wl.new_entries else 0))


# ---------------------------------------------------------------------------
# draws
# ---------------------------------------------------------------------------
def outlier_channels(seed: int) -> np.ndarray:
    return np.sort(_rng(seed, _S_OUTLIER).choice(D_LATENT, OUTLIER_COUNT, replace=False))


def _latent(rng: np.random.Generator, rows: int, outliers: np.ndarray) -> np.ndarray:
    x = rng.standard_normal((rows, D_LATENT), dtype=np.float32)
    x[:, outliers] *= np.float32(OUTLIER_GAIN)
    return x


def kv_latent(wl: Workload, b: int) -> np.ndarray:
    """Main-KV latents of sequence b: float32 [n_entries[b], 512]."""
    return _latent(_rng(wl.seed, _S_KV, 0, b), wl.n_entries[b], outlier_channels(wl.seed))


def index_keys(wl: Workload, b: int) -> np.ndarray:
    """Indexer keys of sequence b: float32 [n_entries[b], 64], N(0,1)."""
    return _rng(wl.seed, _S_IDXK, 0, b).standard_normal((wl.n_entries[b], D_INDEX), dtype=np.float32)


def main_query_bf16(wl: Workload, layer: int, b: int) -> np.ndarray:
    """Main query of sequence b at a layer: bf16 bits (uint16) [T, H, 512], N(0, 1/512)."""
    x = _rng(wl.seed, _S_Q, layer, b).standard_normal((wl.T, wl.H, D_LATENT), dtype=np.float32)
    x *= np.float32(1.0 / np.sqrt(D_LATENT))
    u = x.view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)      # float32 -> bf16, nearest-even
    return ((u + rounding) >> 16).astype(np.uint16)


def index_query(wl: Workload, layer: int, b: int) -> np.ndarray:
    """Indexer query of sequence b at a layer: float32 [T, HI, 64], N(0, 1/64)."""
    x = _rng(wl.seed, _S_IQ, layer, b).standard_normal((wl.T, wl.HI, D_INDEX), dtype=np.float32)
    return x * np.float32(1.0 / np.sqrt(D_INDEX))


def head_weights(wl: Workload, layer: int, b: int) -> np.ndarray:
    """Indexer head weights of sequence b at a layer: float32 [T, HI], U(0, 1)."""
    return _rng(wl.seed, _S_W, layer, b).random((wl.T, wl.HI), dtype=np.float32)


def swa_latent(wl: Workload, layer: int, b: int) -> np.ndarray:
    """Sliding-window token latents of sequence b at a layer: float32 [swa_tokens, 512]."""
    return _latent(_rng(wl.seed, _S_SWA, layer, b), wl.swa_tokens(), outlier_channels(wl.seed))


def window_slot(wl: Workload, b: int, token: int) -> int:
    """Slot of the layer's window buffer that holds absolute token `token` of sequence b.

    Decode keeps a ring of SWA_WINDOW slots, token u in slot u % SWA_WINDOW.  Prefill keeps the
    SWA_WINDOW - 1 tokens before the chunk followed by the chunk, token u in slot
    u - (prefill_start - SWA_WINDOW + 1)."""
    if wl.prefill_start is None:
        return int(token) % SWA_WINDOW
    return int(token) - (wl.prefill_start - (SWA_WINDOW - 1))


def swa_window(wl: Workload, b: int) -> Tuple[np.ndarray, np.ndarray]:
    """(start slot, length) of each query's window inside the layer's window buffer.

    Decode keeps a 128-slot ring: every query sees all filled slots.  Prefill keeps the
    127 tokens before the chunk followed by the chunk; query t sees slots t..t+127."""
    if wl.prefill_start is None:
        n = min(SWA_WINDOW, wl.ctx_tokens[b])
        return np.zeros(wl.T, np.int32), np.full(wl.T, n, np.int32)
    first = wl.prefill_start - (SWA_WINDOW - 1)
    pos = wl.q_pos(b)
    lo = np.maximum(pos - (SWA_WINDOW - 1), 0)
    start = (lo - first).astype(np.int32)
    length = (pos - lo + 1).astype(np.int32)
    return start, length
