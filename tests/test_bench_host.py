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
