"""Host-side helpers of bench.py: the e2e copy grouping and the host page report (no GPU)."""
import ctypes
import mmap

import numpy as np
import torch

import bench


def test_query_copy_groups_cover_every_layer_once_in_order():
    for n in range(0, 13):
        groups = bench.query_copy_groups(n)
        flat = [l for g in groups for l in g]
        assert flat == list(range(n))
        assert all(len(g) == 1 for g in groups[:2])
        assert all(1 <= len(g) <= 2 for g in groups)
    assert bench.query_copy_groups(6) == [[0], [1], [2, 3], [4, 5]]


def test_host_page_report_counts_the_mapping():
    m = mmap.mmap(-1, 8 << 20, flags=mmap.MAP_PRIVATE | mmap.MAP_ANONYMOUS)
    base = ctypes.addressof(ctypes.c_char.from_buffer(m))
    off = (-base) % (2 << 20)
    a = np.frombuffer(m, dtype=np.uint8, count=4 << 20, offset=off)
    a[:] = 1                                           # resident now
    t = torch.from_numpy(a)
    rep = bench.host_page_report([t])
    assert "error" not in rep
    assert rep["rss_kb"] >= 4096                       # the 4 MB touched (the mapping may hold more)
    assert 0 <= rep["anon_huge_kb"] <= rep["rss_kb"]
    assert sum(rep["nodes"].values()) * 4 >= 4096      # pages (4 KB units) on some node
    assert bench.host_page_report([torch.empty(0)]) == {"rss_kb": 0, "anon_huge_kb": 0, "nodes": {}}
    del t, a
    m.close()


def test_attention_traffic_lookup_by_workload():
    """The roofline's measured DRAM traffic is per workload and tied to the kernel source it was
    captured on: a workload with no capture, or a changed source, gives None with a reason."""
    for name in ("decode_128k_b32_F5U", "decode_1m_b4_F5U"):
        got, note = bench.attn_traffic(name)
        assert (got is None and "current kernel source" in note) or (got > 0 and "ncu" in note)
    got, note = bench.attn_traffic("reindex_256k_b16_FIUIUU")
    assert got is None and note == "no capture on this workload"
    saved = bench.ATTN_TRAFFIC_SHA256
    try:
        bench.ATTN_TRAFFIC_SHA256 = "0" * 64
        assert bench.attn_traffic("decode_1m_b4_F5U") == (None, "no capture of the current kernel source")
    finally:
        bench.ATTN_TRAFFIC_SHA256 = saved


def _replica_rank(rank, world, port, out_q):
    import os

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's own total time; the job's time is the slowest rank's
        own_ms = 10.0 + 7.5 * rank
        total = bench.max_over_ranks(torch, dist, own_ms, world, device="cpu")
        out_q.put((rank, total, bench.replica_throughput(32, world, 20, total)))
    finally:
        dist.destroy_process_group()


def test_replica_timing_takes_the_slowest_rank_on_two_gloo_ranks():
    """The multi-GPU bench reports the whole job's queries/s over the slowest rank's time: two gloo
    ranks on the CPU with different totals both see the larger one."""
    import socket

    import torch.multiprocessing as mp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_replica_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, total, value in got:
        assert total == 17.5
        assert value == 32 * 2 * 20 / 17.5e-3
    assert bench.max_over_ranks(torch, None, 3.25, 1) == 3.25       # one rank: no collective
    assert bench.replica_throughput(32, 1, 20, 6.5) == 32 * 20 / 6.5e-3


def test_roofline_work_matches_closed_forms_for_the_decode_workloads():
    """The roofline's numerators (bytes and flops per launch) against the closed forms: per query
    row, K selected rows of 288 B, 128 window rows of 516 B, Q (bf16) and O (bf16) of H x 512,
    K ids and H log-sum-exps; 4 x 512 flop per head and key; the Full indexer reads 36 B per
    visible entry plus H_I x 40 B of query and writes K ids."""
    from compressed_sparse_attention_quantize_b200 import synth
    wl1, wl3 = synth.workload(1), synth.workload(3)
    per_row = 2048 * 288 + 128 * 516 + 64 * 512 * (2 + 2) + 2048 * 4 + 64 * 4
    assert bench.attn_work(wl1, 2) == (32 * per_row, 32 * 64 * (2048 + 128) * 512 * 4)
    assert bench.attn_work(wl3, 2) == (4 * per_row, 4 * 64 * (2048 + 128) * 512 * 4)
    assert bench.attn_work(wl1, 2)[0] == 25452544
    assert bench.index_work(wl1) == 32 * (32768 * 36 + 8 * 40 + 2048 * 4)
    assert wl3.B == 4 and all(131072 <= n <= 262144 for n in wl3.n_entries)
    assert bench.index_work(wl3) == sum(wl3.n_entries) * 36 + 4 * (8 * 40 + 2048 * 4)
