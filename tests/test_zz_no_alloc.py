"""csa2_sparse_attn_noalloc matches csa2_sparse_attn (GPU, through the C ABI).

The no-allocation variant exists for callers that cannot call cudaMalloc: code running under
an allocator that owns the device pool, or a host process that forbids device allocations
once it has started.  Instead of a caller-supplied workspace it keeps the split partials in a
fixed scratch array inside the library.  This test runs the same attention through both entry
points on two different inputs in a row (so the second call meets the first call's leftovers
in the shared scratch) and requires the same results within the parity tolerance.

The file name sorts last so that a run stopping at the first failure has already run every
other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_quantize_b200 as csa2
from compressed_sparse_attention_quantize_b200 import runtime, synth
from tests._parity import check_attention

pytestmark = pytest.mark.gpu


def _rows_beyond_array():
    for rows in range(1, 161):
        if csa2.csa2_sparse_attn_workspace_size(rows, 64, 2048) > (20 << 20):
            return rows
    raise AssertionError("no decode batch up to 160 rows exceeds the no-allocation array")


@pytest.mark.parametrize("B,K", [(4, 256), (32, 2048), ("beyond", 2048)])
def test_noalloc_matches_workspace_entry_point_twice(B, K):
    # 4 rows x 64 heads and top-256 + a 128-token window: several splits per row, so the split
    # partials (the scratch) are really used.  32 rows x top-2048 is the 128K decode shape; the
    # third case takes the fewest rows whose default plan needs more partials than the array
    # holds: the call runs a plan fitted to it.
    if B == "beyond":
        B = _rows_beyond_array()
    wl = synth.scaled(synth.workload(1), B=B, n=3000, K=K, name="noalloc")
    r = runtime.GroupRunner(wl, layers=2)
    r.run()
    torch.cuda.synchronize()
    idx = r.layer_data[0]["idx"]
    cnt = (idx >= 0).sum(dim=1).to(torch.int32)
    ws_bytes = csa2.csa2_sparse_attn_workspace_size(r.rows, wl.H, wl.K)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device="cuda")
    for layer in (0, 1):
        ld = r.layer_data[layer]
        args = (ld["q"], wl.B, wl.T, wl.H, 512, r.kv, 288, r.seq_start, r.n_entries, idx, cnt, wl.K,
                ld["swa_codes"], ld["swa_scale"], r.swa_cap, r.swa_start, r.swa_len, r.softmax_scale)
        out_ref = torch.empty((r.rows, wl.H, 512), dtype=torch.float32, device="cuda")
        lse_ref = torch.empty((r.rows, wl.H), dtype=torch.float32, device="cuda")
        csa2.csa2_sparse_attn(*args, out_ref, csa2.DTYPE_F32, lse_ref, ws, ws_bytes)
        out = torch.full((r.rows, wl.H, 512), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((r.rows, wl.H), float("nan"), dtype=torch.float32, device="cuda")
        csa2.csa2_sparse_attn_noalloc(*args, out, csa2.DTYPE_F32, lse)
        torch.cuda.synchronize()
        for row in range(r.rows):
            check_attention(out[row].cpu().numpy(), out_ref[row].cpu().numpy(), f"layer {layer} row {row}")
        assert np.allclose(lse.cpu().numpy(), lse_ref.cpu().numpy(), rtol=0, atol=1e-3)
    assert csa2.csa2_device_error() == 0
