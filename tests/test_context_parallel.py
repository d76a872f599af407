"""Context-parallel decode (one sequence's entries split across ranks).

CPU: two gloo ranks run the decomposition (shard top-K with scores, all-gather, merged top-K,
shard attention, all-gather, log-sum-exp merge) with the oracle as each rank's local compute,
and must reproduce the single-process oracle on the whole sequence: the same selected sets
(bit-exact) and the same outputs.  GPU: the CUDA path of every step, with two shards run one
after the other on one GPU and the exchanges done by stacking, against the same oracle.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_attention_quantize_b200 import synth
from tests._cp_oracle import OracleShard, shard_bounds
from tests._parity import OracleSeq, check_attention


def _workload():
    return synth.scaled(synth.workload(3), B=2, n=[2600, 1900], K=96, H=16, name="cp")


def _reference(wl, seqs, layers, scale):
    """Whole-sequence oracle: Full in layer 0, Reuse after."""
    res = []
    for b in range(wl.B):
        os_ = seqs[b]
        L = os_.layer(0)
        idx, cnt, _, _, _ = oracle.full_index(L["qc"][0], L["qs"][0], L["w"][0], os_.k_codes, os_.k_scales,
                                              wl.n_entries[b], wl.K)
        outs = [os_.attention(l, 0, idx, scale) for l in range(layers)]
        res.append((idx, cnt, outs))
    return res


def _rank(rank, world, port, out_q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from compressed_sparse_attention_quantize_b200.context_parallel import Comm
        comm = Comm()
        wl = _workload()
        scale = 1.0 / np.sqrt(512)
        seqs = [OracleSeq(wl, b) for b in range(wl.B)]
        sh = OracleShard(wl, seqs, rank, world, scale)
        results = []
        prev = None
        for l in range(3):
            if l == 0:
                scores, ids, cnt = sh.local_topk(l)
                prev = sh.merge_topk(comm.all_gather(scores), comm.all_gather(ids), comm.all_gather(cnt),
                                     comm.all_gather(sh.shard_lo))
            out_l, lse_l = sh.attention(l, *prev)
            out, lse = sh.merge_attention(comm.all_gather(out_l), comm.all_gather(lse_l))
            results.append((prev[0].numpy().copy(), prev[1].numpy().copy(), out, lse))
        if rank == 0:
            out_q.put(results)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_whole_sequence_oracle():
    import socket
    import torch.multiprocessing as mp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = q.get(timeout=600)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    wl = _workload()
    scale = 1.0 / np.sqrt(512)
    seqs = [OracleSeq(wl, b) for b in range(wl.B)]
    ref = _reference(wl, seqs, 3, scale)
    for l, (idx, cnt, out, lse) in enumerate(results):
        for b in range(wl.B):
            ridx, rcnt, routs = ref[b]
            assert int(cnt[b]) == rcnt and np.array_equal(idx[b], ridx), (l, b)
            rout, rlse = routs[l]
            assert np.allclose(out[b], rout, rtol=1e-9, atol=1e-12), (l, b)
            assert np.allclose(lse[b], rlse, rtol=1e-12, atol=1e-12), (l, b)


def test_shard_bounds_partition():
    for n in (0, 1, 7, 1000, 262144):
        for G in (1, 2, 3, 8):
            edges = [shard_bounds(n, g, G) for g in range(G)]
            assert edges[0][0] == 0 and edges[-1][1] == n
            assert all(edges[g][1] == edges[g + 1][0] for g in range(G - 1))


@pytest.mark.gpu
def test_device_shards_match_whole_sequence_oracle():
    """CUDA steps for 2 shards on one GPU (run in turn; exchanges by stacking) vs the oracle."""
    import compressed_sparse_attention_quantize_b200 as csa2
    from compressed_sparse_attention_quantize_b200 import runtime
    from compressed_sparse_attention_quantize_b200.context_parallel import DeviceShard, LayerInputs
    wl = _workload()
    G = 2
    scale = 1.0 / np.sqrt(512)
    seqs = [OracleSeq(wl, b) for b in range(wl.B)]
    ref = _reference(wl, seqs, 2, scale)
    dev = torch.device("cuda")
    shards, layer_inputs = [], []
    for g in range(G):
        bounds = [shard_bounds(n, g, G) for n in wl.n_entries]
        ns = [hi - lo for lo, hi in bounds]
        starts = np.concatenate([[0], np.cumsum(ns)[:-1]]).astype(np.int64)
        total = max(int(sum(ns)), 1)
        kv = torch.zeros((total, 288), dtype=torch.uint8, device=dev)
        kc = torch.zeros((total, 32), dtype=torch.uint8, device=dev)
        ks = torch.zeros((total, 4), dtype=torch.uint8, device=dev)
        for b, (lo, hi) in enumerate(bounds):
            lat = torch.from_numpy(synth.kv_latent(wl, b)[lo:hi]).to(dev)
            runtime.quantize_fp4_rows(lat, kv[starts[b]:], kv[starts[b]:, 256:], 288, 288)
            ik = torch.from_numpy(synth.index_keys(wl, b)[lo:hi]).to(dev)
            runtime.quantize_fp4_rows(ik, kc[starts[b]:], ks[starts[b]:], 32, 4)
        sh = DeviceShard(kv, kc, ks, torch.from_numpy(starts).to(dev),
                         torch.tensor([lo for lo, _ in bounds], dtype=torch.int64, device=dev),
                         torch.tensor(ns, dtype=torch.int32, device=dev), wl.B, 1, wl.H, wl.HI, wl.K,
                         wl.swa_tokens(), scale)
        shards.append(sh)
        per_layer = []
        for l in range(2):
            q = np.stack([synth.main_query_bf16(wl, l, b) for b in range(wl.B)]).reshape(wl.B, wl.H, 512)
            iq = np.stack([synth.index_query(wl, l, b) for b in range(wl.B)]).reshape(wl.B * wl.HI, 64)
            iqc = torch.empty((wl.B * wl.HI, 32), dtype=torch.uint8, device=dev)
            iqs = torch.empty((wl.B * wl.HI, 4), dtype=torch.uint8, device=dev)
            runtime.quantize_fp4_rows(torch.from_numpy(iq).to(dev), iqc, iqs, 32, 4)
            w = np.stack([synth.head_weights(wl, l, b) for b in range(wl.B)]).reshape(wl.B, wl.HI)
            sw = np.stack([synth.swa_latent(wl, l, b) for b in range(wl.B)]).reshape(wl.B * wl.swa_tokens(), 512)
            swc = torch.empty((wl.B * wl.swa_tokens(), 512), dtype=torch.uint8, device=dev)
            sws = torch.empty((wl.B * wl.swa_tokens(),), dtype=torch.float32, device=dev)
            runtime.quantize_fp8_rows(torch.from_numpy(sw).to(dev), swc, sws)
            st, ln = zip(*[synth.swa_window(wl, b) for b in range(wl.B)])
            lens = np.concatenate(ln).astype(np.int32) if g == G - 1 else np.zeros(wl.B, np.int32)
            per_layer.append(LayerInputs(
                q=torch.from_numpy(q.view(np.int16)).to(dev), swa_codes=swc, swa_scale=sws,
                swa_start=torch.from_numpy(np.concatenate(st).astype(np.int32)).to(dev),
                swa_len=torch.from_numpy(lens).to(dev), iq_codes=iqc, iq_scales=iqs,
                iw=torch.from_numpy(np.ascontiguousarray(w, np.float32)).to(dev)))
        layer_inputs.append(per_layer)
    # layer 0 (Full): shard top-K with scores, "all-gather" by stacking, merged top-K
    parts = [shards[g].local_topk(layer_inputs[g][0]) for g in range(G)]
    scores_g = torch.stack([p[0] for p in parts])
    ids_g = torch.stack([p[1] for p in parts])
    cnt_g = torch.stack([p[2] for p in parts])
    lo_g = torch.stack([sh.shard_lo for sh in shards])
    idx, cnt = shards[0].merge_topk(scores_g, ids_g, cnt_g, lo_g)
    torch.cuda.synchronize()
    for b in range(wl.B):
        ridx, rcnt, _ = ref[b]
        assert int(cnt[b]) == rcnt and np.array_equal(idx[b].cpu().numpy(), ridx), b
    # layers 0 and 1 attention (layer 1 reuses the selection)
    for l in range(2):
        res = [shards[g].attention(layer_inputs[g][l], idx, cnt) for g in range(G)]
        out, lse = shards[0].merge_attention(torch.stack([x[0] for x in res]), torch.stack([x[1] for x in res]))
        torch.cuda.synchronize()
        for b in range(wl.B):
            rout, rlse = ref[b][2][l]
            check_attention(out[b].cpu().numpy(), rout, f"layer {l} seq {b}")
            assert np.allclose(lse[b].cpu().numpy(), rlse, rtol=1e-4, atol=1e-4)
