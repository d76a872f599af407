#!/usr/bin/env python
"""CSA2 hot-path benchmark: decode queries/s of one CSA2 layer group on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl csa2|reference] [--config C]

One step = one decode token of every sequence of the workload through the whole hot path: the
step's quantise-on-write, then the layer group (indexer + top-K of the Full layer, Reindex
re-scoring where the mode table has it, and attention of every layer).  Default workload:
decode at 128K context, batch 32, 1 Full + 5 Reuse layers (the headline line).  The same line
carries, under "workloads", the same measurement of the other timed workloads: decode at 1M
context (batch 4), the Reindex group at 256K (batch 16) and the prefill chunk (4096 queries).

Printed (rank 0, one JSON line): value = queries/s over all ranks (device time, CUDA events on
the launch stream, L2 flushed by a 256 MB write between steps, max over ranks); e2e = the same
metric through csa2_layer_group with host buffers (host->device copies of the step's inputs and
the device->host read of the last layer's output inside the timed region); roofline of the
dominant kernel; cpu_baseline = the oracle on the host cores over a bounded sample.

With --gpus N > 1 (torchrun) every rank runs its own replica of the workload (independent
sequences; the decode path has no exchange step), so scaling is weak.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "CSA2 decode queries/sec at 128K and 1M ctx; achieved HBM GB/s vs ~8 TB/s"
UNIT = "queries/s"
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------------------------------
# algorithmic work per call (bytes that must move; flops of the contraction)
# ------------------------------------------------------------------------------------------
# DRAM bytes (read + write) of one attn_tc_kernel launch per decode workload, each from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum), together with the SHA-256 of the kernel
# source they were taken on: when the source has changed since, the figures are stale and the
# line reports traffic null.
ATTN_TRAFFIC_SHA256 = "3e6a7affcd4af519d0fbc9da779944ec81806f7a7b723d8fb2c6e95a1026f79b"
ATTN_TRAFFIC = {
    "decode_128k_b32_F5U": {
        "bytes": 28974848 + 140288,
        "capture": "ncu --set full --clock-control none -k 'regex:attn_tc_kernel|attn_tc_merge' "
                   "-s 8 -c 3 python bench.py --config 1 --entries 16384 --steps 2 --warmup 3 --quick "
                   "--no-cpu-baseline --eager (dram__bytes_read.sum + dram__bytes_write.sum of attn_tc_kernel; "
                   "the attention's bytes do not depend on the entry count)"},
    "decode_1m_b4_F5U": {
        "bytes": 3815296,                       # read 3817472 and 3813120, written 0
        "capture": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                   "--clock-control none -k regex:attn_tc_kernel -s 6 -c 2 python bench.py --config 3 "
                   "--steps 3 --warmup 3 --quick --no-cpu-baseline --eager (mean of the two launches' "
                   "dram__bytes_read.sum + dram__bytes_write.sum)"},
}
ATTN_SOURCE = os.path.join(ROOT, "compressed_sparse_attention_quantize_b200", "csrc", "attn_tc.cu")


def attn_traffic(workload):
    """(bytes or None, note): the captured DRAM traffic of one attention launch on `workload` if
    it was taken on the current kernel source."""
    import hashlib
    rec = ATTN_TRAFFIC.get(workload)
    if rec is None:
        return None, "no capture on this workload"
    try:
        with open(ATTN_SOURCE, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None, "kernel source not found"
    if sha != ATTN_TRAFFIC_SHA256:
        return None, "no capture of the current kernel source"
    return rec["bytes"], rec["capture"]


def visible_counts(wl, b):
    """Entries each query of sequence b can select, for the byte and flop accounting: entry j
    covers tokens 4j..4j+3 and is visible at token p when 4j + 3 <= p (decode: all)."""
    import numpy as np
    if wl.prefill_start is None:
        return np.array([wl.n_entries[b]], np.int64)
    return np.minimum((wl.q_pos(b) + 1) // 4, wl.n_entries[b])


STEP_WRITES = ("quantise-on-write inside the step: the newest compressed entry (FP4) and its indexer "
               "key (FP4) of every sequence, every Full/Reindex layer's indexer query (FP4), every "
               "layer's window entry of the step token (E4M3); an entry is written every step, an "
               "upper bound on the one completed every 4th token")


def write_calls(runner):
    """Library calls of one write_step(): one csa2_quantize_kv_batch launch."""
    return 1 if (runner.entry_jobs or runner.window_jobs or runner.query_jobs) else 0


def write_work(runner):
    """Bytes of one write_step(): float rows and destination rows read, quantised rows written."""
    byts = 0
    if runner.step_rows is not None:
        m = runner.step_rows.numel()
        byts += m * (512 * 4 + 288 + 8) + m * (64 * 4 + 36 + 8)
    if runner.step_win_rows is not None:
        byts += runner.step_win_rows.numel() * (512 * 4 + 516 + 8)
    for ld in runner.layer_data:
        if "iq_f32" in ld:
            byts += ld["iq_f32"].shape[0] * (64 * 4 + 36)
    return byts


def attn_work(wl, out_bytes):
    """Bytes and flops of one csa2_sparse_attn call over the workload."""
    from compressed_sparse_attention_quantize_b200 import synth
    byts = 0
    flops = 0
    for b in range(wl.B):
        nvis = visible_counts(wl, b)
        _, swl = synth.swa_window(wl, b)
        for t in range(wl.T):
            sel = min(wl.K, int(nvis[t]))
            keys = sel + int(swl[t])
            byts += sel * 288 + int(swl[t]) * 516 + wl.H * 512 * (2 + out_bytes) + wl.K * 4 + wl.H * 4
            flops += wl.H * keys * 512 * 4
    return byts, flops


def index_work(wl):
    """Bytes of one Full-mode csa2_index_topk call (keys scanned + queries + selection written)."""
    byts = 0
    for b in range(wl.B):
        nvis = visible_counts(wl, b)
        for t in range(wl.T):
            byts += int(nvis[t]) * 36 + wl.HI * 40 + wl.K * 4
            if wl.P:
                byts += wl.P * 4
    return byts


def reindex_work(wl):
    """Bytes of one Reindex csa2_index_topk call (pool ids and the gathered keys they name,
    queries, selection written)."""
    byts = 0
    for b in range(wl.B):
        nvis = visible_counts(wl, b)
        for t in range(wl.T):
            pool = min(wl.P, int(nvis[t]))
            byts += pool * (4 + 36) + wl.HI * 40 + wl.K * 4
    return byts


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        self.f.close()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        power = [num(r[3]) or 0.0 for r in rows]
        pmax = max(power) if power else 0.0
        loaded = [num(r[1]) for r, p in zip(rows, power) if p >= 0.5 * pmax and num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded or sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": reasons, "samples": len(rows),
                "power_w_max": pmax}


# ------------------------------------------------------------------------------------------
# reference arm / CPU baseline: the oracle on the host cores
# ------------------------------------------------------------------------------------------
def oracle_sample(wl, rows, softmax_scale):
    """Run the oracle over `rows` query rows (setup outside, returns elapsed seconds of the
    per-query work: indexer scores, top-K, pool/Reindex, attention of every layer)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from tests._parity import OracleSeq
    seqs = {}
    for r in rows:
        b, t = divmod(r, wl.T)
        if b not in seqs:
            s = OracleSeq(wl, b)
            for l in range(len(wl.modes)):
                s.layer(l)
            seqs[b] = s
    t0 = time.perf_counter()
    for r in rows:
        b, t = divmod(r, wl.T)
        sel = seqs[b].indices(t, wl.modes)
        for l in range(len(wl.modes)):
            seqs[b].attention(l, t, sel[l][0], softmax_scale)
    return time.perf_counter() - t0


def cpu_baseline(wl, softmax_scale, budget_s=15.0):
    import oracle
    oracle.build()
    t1 = oracle_sample(wl, [0], softmax_scale)
    n = max(1, min(wl.B * wl.T, int(budget_s / max(t1, 1e-3))))
    rows = list(range(1, 1 + n)) if n + 1 <= wl.B * wl.T else list(range(n))
    el = oracle_sample(wl, rows, softmax_scale)
    return {"value": len(rows) / el, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(rows)} query rows of '{wl.name}' through all {len(wl.modes)} layers "
                      f"(indexer over every visible entry, top-K, attention per layer); "
                      f"oracle-side cache quantisation not timed"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    scale = 1.0 / math.sqrt(512)
    # one step = a bounded sample of the workload (a single query row through every layer)
    for w in range(args.warmup):
        oracle_sample(wl, [w % (wl.B * wl.T)], scale)
    tot = 0.0
    for k in range(args.steps):
        tot += oracle_sample(wl, [k % (wl.B * wl.T)], scale)
    value = args.steps / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64/f32 (oracle)", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.B, "ctx_tokens": wl.ctx_tokens[0],
                       "layers": ",".join(wl.modes), "heads": wl.H, "topk": wl.K,
                       "step": "one query row through every layer (bounded sample)"},
            "cpu_baseline": {"kind": "oracle", "cores": oracle.num_threads(), "value": value,
                             "unit": UNIT, "sample": "one query row per step through every layer"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------
# the CUDA arm
# ------------------------------------------------------------------------------------------
def time_steps(torch, step, steps, flush):
    """Per-step CUDA-event times (ms) with an L2 flush before every step (outside the events)."""
    st = torch.cuda.current_stream()
    evs = []
    for _ in range(steps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(st)
        step()
        e1.record(st)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def breakdown(torch, csa2, runner, steps, flush, writes=False):
    """Per-call device times of the decomposed step: the step's writes (one csa2_quantize_kv_batch
    launch, replayed from a one-node CUDA graph so that host launch overhead is not counted),
    then csa2_index_topk + csa2_sparse_attn per layer."""
    wl = runner.wl
    dev = runner.workspace.device
    rows = runner.rows
    idx = torch.empty((rows, wl.K), dtype=torch.int32, device=dev)
    cnt = torch.empty((rows,), dtype=torch.int32, device=dev)
    P = wl.P if "I" in runner.modes else 0
    pool = torch.empty((rows, max(P, 1)), dtype=torch.int32, device=dev)
    pool_len = torch.empty((rows,), dtype=torch.int32, device=dev)
    iws_bytes = max(csa2.csa2_index_topk_workspace_size(0, rows, runner.max_n, wl.K, P),
                    csa2.csa2_index_topk_workspace_size(1, rows, runner.max_n, wl.K, max(P, 1)))
    iws = torch.empty((iws_bytes,), dtype=torch.uint8, device=dev)
    aws_bytes = csa2.csa2_sparse_attn_workspace_size(rows, wl.H, wl.K)
    aws = torch.empty((aws_bytes,), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    write_graph = floor_graph = None
    if writes:
        runner.write_step()
        torch.cuda.synchronize()
        write_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(write_graph):
            runner.write_step()
        # the same measurement of a one-element add: what any one-node graph costs here
        one = torch.zeros((1,), dtype=torch.float32, device=dev)
        one.add_(1.0)
        torch.cuda.synchronize()
        floor_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(floor_graph):
            one.add_(1.0)
        torch.cuda.synchronize()
    times = {"step_writes": [], "graph_floor": [], "index_topk": [], "reindex_topk": [], "sparse_attn": []}
    for _ in range(steps):
        flush()
        marks = []
        def ev():
            e = torch.cuda.Event(enable_timing=True)
            e.record(st)
            return e
        if write_graph is not None:
            e0 = ev()
            write_graph.replay()
            marks.append(("step_writes", e0, ev()))
            flush()
            e0 = ev()
            floor_graph.replay()
            marks.append(("graph_floor", e0, ev()))
            flush()
        for l, m in enumerate(runner.modes):
            ld = runner.layer_data[l]
            if m != "U":
                e0 = ev()
                if m == "F":
                    csa2.csa2_index_topk(0, ld["iq_codes"], ld["iq_scales"], ld["iw"], wl.B, wl.T, wl.HI,
                                         runner.k_codes, 32, runner.k_scales, 4, runner.seq_start,
                                         runner.n_entries, runner.max_n, runner.q_pos, None, None, 0,
                                         wl.K, idx, cnt, P, pool if P else None, pool_len if P else None,
                                         iws, iws_bytes)
                    marks.append(("index_topk", e0, ev()))
                else:
                    csa2.csa2_index_topk(1, ld["iq_codes"], ld["iq_scales"], ld["iw"], wl.B, wl.T, wl.HI,
                                         runner.k_codes, 32, runner.k_scales, 4, runner.seq_start,
                                         runner.n_entries, runner.max_n, runner.q_pos, pool, pool_len, P,
                                         wl.K, idx, cnt, 0, None, None, iws, iws_bytes)
                    marks.append(("reindex_topk", e0, ev()))
            e0 = ev()
            csa2.csa2_sparse_attn(ld["q"], wl.B, wl.T, wl.H, 512, runner.kv, 288, runner.seq_start,
                                  runner.n_entries, idx, cnt,
                                  wl.K, ld["swa_codes"], ld["swa_scale"], runner.swa_cap, runner.swa_start,
                                  runner.swa_len, runner.softmax_scale, ld["out"], runner.out_dtype, ld["lse"],
                                  aws, aws_bytes)
            marks.append(("sparse_attn", e0, ev()))
        torch.cuda.synchronize()
        for name, a, b in marks:
            times[name].append(a.elapsed_time(b))
    del write_graph, floor_graph
    return {k: v for k, v in times.items() if v}


class gpu_local_cpus:
    """Run the enclosed code on the CPUs NVML reports as local to the current GPU (read-only
    NVML query), then restore the affinity.  Page-locked buffers allocated and first touched
    inside land on the GPU's NUMA node, which decides the host<->device copy bandwidth."""

    def __init__(self, torch):
        self.torch = torch
        self.saved = None
        self.used = False

    def __enter__(self):
        try:
            import pynvml
            props = self.torch.cuda.get_device_properties(self.torch.cuda.current_device())
            busid = f"{props.pci_domain_id:04x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByPciBusId(busid)
            words = (os.cpu_count() + 63) // 64
            mask = pynvml.nvmlDeviceGetCpuAffinity(h, words)
            cpus = {w * 64 + b for w, m in enumerate(mask) for b in range(64) if (int(m) >> b) & 1}
            cpus &= set(os.sched_getaffinity(0))
            if cpus:
                self.saved = os.sched_getaffinity(0)
                os.sched_setaffinity(0, cpus)
                self.used = True
        except Exception:
            self.saved = None
        return self

    def __exit__(self, *exc):
        if self.saved is not None:
            os.sched_setaffinity(0, self.saved)
        return False


def host_page_report(tensors):
    """How the host buffers are backed, from /proc/self/smaps and numa_maps (read-only): resident
    and transparent-huge-page kB, and pages per NUMA node, over the mappings that hold them."""
    ranges = [(t.data_ptr(), t.data_ptr() + t.numel() * t.element_size()) for t in tensors if t.numel()]
    rep = {"rss_kb": 0, "anon_huge_kb": 0, "nodes": {}}
    try:
        vmas = set()
        cur = None
        with open("/proc/self/smaps") as f:
            for line in f:
                head = line.split()
                if "-" in head[0] and len(head) >= 5 and all(c in "0123456789abcdef-" for c in head[0]):
                    lo, hi = (int(x, 16) for x in head[0].split("-"))
                    cur = (lo, hi) if any(a < hi and b > lo for a, b in ranges) else None
                    if cur:
                        vmas.add(cur)
                elif cur and head[0] == "Rss:":
                    rep["rss_kb"] += int(head[1])
                elif cur and head[0] == "AnonHugePages:":
                    rep["anon_huge_kb"] += int(head[1])
        starts = {lo for lo, _ in vmas}
        with open("/proc/self/numa_maps") as f:
            for line in f:
                parts = line.split()
                if int(parts[0], 16) in starts:
                    for tok in parts[2:]:
                        if tok.startswith("N") and "=" in tok:
                            node, n = tok.split("=")
                            rep["nodes"][node] = rep["nodes"].get(node, 0) + int(n)
    except (OSError, ValueError, IndexError) as exc:
        rep["error"] = f"{type(exc).__name__}: {exc}"[:120]
    return rep


def topk_side_reference(torch, csa2, wl, flush, reps=10):
    """torch.topk next to the library's top-K on the same fp32 score buffer (side reference only).

    Scores: [rows][n] uniform on [0, 1), seeded; K of n per row.  The library's side is
    csa2_topk_merge_shards with one shard holding the whole row (it selects from the list in
    place with the cluster top-K kernel, one launch), which also returns the selection in
    ascending index order.  Both selections are checked to have the same K-th largest score
    per row."""
    rows, n, K = wl.B * wl.T, int(max(wl.n_entries)), wl.K
    g = torch.Generator(device="cuda")
    g.manual_seed(int(wl.seed) + 77)
    scores = torch.rand((1, rows, n), generator=g, device="cuda", dtype=torch.float32)
    ids = torch.arange(n, dtype=torch.int32, device="cuda").repeat(1, rows, 1).contiguous()
    cnt = torch.full((1, rows), n, dtype=torch.int32, device="cuda")
    idx = torch.empty((rows, K), dtype=torch.int32, device="cuda")
    out_cnt = torch.empty((rows,), dtype=torch.int32, device="cuda")
    ws = torch.empty(csa2.csa2_topk_merge_shards_workspace_size(1, rows, n), dtype=torch.uint8, device="cuda")
    res = {}

    def ours():
        csa2.csa2_topk_merge_shards(scores, ids, None, cnt, 1, rows, n, K, idx, out_cnt, ws, ws.numel())

    def theirs():
        res["t"] = torch.topk(scores[0], K, dim=1, sorted=False)

    for f in (ours, theirs):
        f()
    t_ours = time_steps(torch, ours, reps, flush)
    t_torch = time_steps(torch, theirs, reps, flush)
    kth_ours = scores[0].gather(1, idx.long()).min(dim=1).values
    kth_torch = res["t"].values.min(dim=1).values
    return {"scores": f"[{rows}][{n}] fp32 uniform [0,1)", "k": K,
            "csa2_topk_ms": statistics.median(t_ours), "torch_topk_ms": statistics.median(t_torch),
            "kth_value_equal": bool(torch.equal(kth_ours, kth_torch)),
            "note": "csa2_topk_merge_shards (one shard) vs torch.topk(sorted=False); L2 flushed before each call"}


def query_copy_groups(n_layers):
    """The layers whose main queries cross in one copy, in order: the first two layers alone, then
    pairs ([0], [1], [2, 3], [4, 5], ...): fewer copies, while the first layers' queries land early."""
    groups, l = [], 0
    while l < n_layers:
        n = 1 if l < 2 else 2
        groups.append(list(range(l, min(n_layers, l + n))))
        l += n
    return groups


def e2e_measure(torch, csa2, runner, steps, warmup, flush, writes=False):
    """The metric through csa2_layer_group with host buffers.  Per step: every layer's main query
    (bf16) and indexer query/weights (fp32) are copied from pinned host memory on a copy stream,
    layer by layer (the indexer queries are quantised there too; with ``writes`` the step's new
    entry and window latents are copied and quantised there as well), and each layer of the group
    waits only for its own inputs (the group's per-layer ready events), so the copies of later
    layers overlap the work of earlier ones; the last layer's output is read back at the end.
    Steps do not overlap: the copy stream starts a step after the previous step's work."""
    from compressed_sparse_attention_quantize_b200 import runtime, synth
    wl = runner.wl
    class Stage:
        """Several inputs in one host buffer from the library's allocator (csa2_host_alloc:
        page-locked, 2 MB pages; copies from 4 KB-page buffers ran at 32 GB/s and slowed the group
        beside them by 10-50 %) and one device buffer, so that they cross in one copy (every copy
        pays a fixed cost before its first byte lands)."""

        def __init__(self, parts):
            offs, n = [], 0
            for _, t in parts:
                offs.append(n)
                n += (t.numel() * t.element_size() + 255) // 256 * 256
            self.host = csa2.host_empty((n,), torch.uint8)
            self.dev = torch.empty((n,), dtype=torch.uint8, device="cuda")
            self.views, self.bytes, self.span = {}, 0, {}
            for (name, t), o in zip(parts, offs):
                nb = t.numel() * t.element_size()
                self.host[o:o + nb].view(t.dtype).view(t.shape).copy_(t)
                self.views[name] = self.dev[o:o + nb].view(t.dtype).view(t.shape)
                self.span[name] = (o, o + nb)
                self.bytes += nb

        def copy(self, first=None, last=None):
            """One copy of all parts, or of the parts from `first` through `last`."""
            if first is None:
                self.dev.copy_(self.host, non_blocking=True)
            else:
                lo, hi = self.span[first][0], self.span[last][1]
                self.dev[lo:hi].copy_(self.host[lo:hi], non_blocking=True)

    h2d = 0
    L = len(runner.modes)
    stages = [None] * L                      # per layer: its indexer inputs (+ the new entries)
    with gpu_local_cpus(torch) as local:
        for l, m in enumerate(runner.modes):
            ld = runner.layer_data[l]
            parts = []
            if m != "U":
                iq = np.stack([synth.index_query(wl, l, b) for b in range(wl.B)]).reshape(-1, 64)
                parts += [("iq", torch.from_numpy(iq)), ("iw", ld["iw"].cpu())]
            if l == 0 and writes and runner.step_rows is not None:
                parts += [("kv", runner.step_kv.cpu()), ("ik", runner.step_ik.cpu())]
            if parts:
                stages[l] = Stage(parts)
                h2d += stages[l].bytes
        # the window tokens and every layer's main query in one buffer, copied in groups that grow
        # along the layers: [window, q0], [q1], [q2, q3], [q4, q5], ...: fewer copies (each has a
        # fixed cost), while the first layers still get their query early
        has_win = writes and runner.step_win_rows is not None
        bulk = Stage(([("win", runner.step_win_lat.cpu())] if has_win else [])
                     + [(f"q{l}", runner.layer_data[l]["q"].cpu()) for l in range(L)])
        h2d += bulk.bytes
        groups = query_copy_groups(L)
        out_last = runner.layer_data[-1]["out"]
        out_host = csa2.host_empty(out_last.shape, out_last.dtype)
    pages = host_page_report([bulk.host] + [st.host for st in stages if st is not None] + [out_host])
    d2h = out_host.numel() * out_host.element_size()
    # quantise-on-write jobs and indexer weights read the device halves of the stages
    st0 = stages[0]
    entry_jobs, window_jobs, query_jobs = runner.write_jobs(
        kv=st0.views.get("kv") if st0 else None, ik=st0.views.get("ik") if st0 else None,
        win=bulk.views["win"] if has_win else None,
        iq=[st.views["iq"] if st is not None and "iq" in st.views else None for st in stages])
    qjob = iter(query_jobs)
    stage_jobs = []
    for l, m in enumerate(runner.modes):
        jobs = [next(qjob)] if m != "U" else []
        if l == 0 and writes:
            jobs += entry_jobs
        stage_jobs.append(jobs)
    saved_iw = [d.iw for d in runner.layer_descs]
    saved_q = [d.q for d in runner.layer_descs]
    for l, st in enumerate(stages):
        if st is not None and "iw" in st.views:
            runner.layer_descs[l].iw = st.views["iw"].data_ptr()
    for l in range(L):
        runner.layer_descs[l].q = bulk.views[f"q{l}"].data_ptr()
    group_of = {g[0]: g for g in groups}
    cur = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream()
    ready = [torch.cuda.Event() for _ in runner.modes]
    attn_ready = [torch.cuda.Event() for _ in runner.modes]
    for ev in ready + attn_ready:
        ev.record(cur)                       # creates the handles
    runner.set_layer_events([ev.cuda_event for ev in ready], None, [ev.cuda_event for ev in attn_ready])

    def body(main):
        copy_stream.wait_stream(main)
        with torch.cuda.stream(copy_stream):
            for l, m in enumerate(runner.modes):
                # a layer's indexer inputs first, and before the first layer the step's new
                # entries (the indexer scores them), in one copy: the indexer starts while the
                # main query and the window tokens, which only the attention needs, are still
                # being copied
                if stages[l] is not None:
                    stages[l].copy()
                if stage_jobs[l]:
                    csa2.csa2_quantize_kv_batch(stage_jobs[l], stream=copy_stream)
                ready[l].record(copy_stream)
                if l in group_of:                     # this layer starts a group of main queries
                    g = group_of[l]
                    first = "win" if (l == 0 and has_win) else f"q{g[0]}"
                    bulk.copy(first, f"q{g[-1]}")
                    if first == "win":
                        csa2.csa2_quantize_kv_batch(window_jobs, stream=copy_stream)
                attn_ready[l].record(copy_stream)
        runner.run()
        out_host.copy_(out_last, non_blocking=True)

    def copies_only():
        """The step's host->device and device->host copies alone (same buffers, same order)."""
        for l in range(L):
            if stages[l] is not None:
                stages[l].copy()
            if l in group_of:
                g = group_of[l]
                bulk.copy("win" if (l == 0 and has_win) else f"q{g[0]}", f"q{g[-1]}")
        out_host.copy_(out_last, non_blocking=True)

    graph = None
    try:
        copies_only()
        torch.cuda.synchronize()
        copy_ms = statistics.median(time_steps(torch, copies_only, max(3, steps), lambda: None))
        for _ in range(warmup):
            flush()
            body(cur)
        torch.cuda.synchronize()
        # the whole step (both streams, copies included) as one CUDA graph, as the device step is
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                body(torch.cuda.current_stream())
            torch.cuda.synchronize()
            graph = g
        except Exception:                  # capture refused: time the eager step instead
            torch.cuda.synchronize()
        step = graph.replay if graph is not None else (lambda: body(cur))
        for _ in range(2):
            flush()
            step()
        torch.cuda.synchronize()
        ms = time_steps(torch, step, steps, flush)
    finally:
        torch.cuda.synchronize()
        runner.set_layer_events(None, None)
        for d, p, pq in zip(runner.layer_descs, saved_iw, saved_q):
            d.iw, d.q = p, pq
    return {"value": runner.rows * steps / (sum(ms) / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": sum(ms) / steps,
            "ms_per_step_min_median_max": [min(ms), statistics.median(ms), max(ms)],
            "overlap": "input copies on a second stream: per layer its indexer inputs (and, before the first "
                       "layer, the step's new entries) in one copy; the window tokens and main queries in "
                       "growing groups [window, q0], [q1], [q2, q3], ...",
            "copies_per_step": sum(st is not None for st in stages) + len(groups) + 1,
            "copy_ms_per_step": copy_ms, "copy_gbs": (h2d + d2h) / (copy_ms * 1e-3) / 1e9,
            "copy_note": "the step's copies alone, back to back on one stream (no kernels)",
            "step": "cuda graph" if graph is not None else "eager",
            "host_buffers": "csa2_host_alloc (page-locked, 2 MB pages requested), "
                            + ("allocated on the GPU's local CPUs" if local.used else "default placement"),
            "host_pages": pages}


def kernel_table(wl, runner, bd, peaks, out_bytes):
    """Per-call times, algorithmic bytes/flops and HBM fractions of the decomposed step."""
    hbm_peak = peaks[0]
    ab, af = attn_work(wl, out_bytes)
    kernels = {}
    if "sparse_attn" in bd:
        t_ms = statistics.mean(bd["sparse_attn"])
        kernels["sparse_attn"] = {"launches_per_step": len(runner.modes), "avg_ms": t_ms,
                                  "algorithmic_bytes": ab, "algorithmic_flops": af,
                                  "achieved_gbs": ab / (t_ms * 1e-3) / 1e9,
                                  "achieved_tflops": af / (t_ms * 1e-3) / 1e12}
    if "step_writes" in bd:
        t_ms = statistics.mean(bd["step_writes"])
        wb = write_work(runner)
        kernels["step_writes"] = {"launches_per_step": 1, "calls": write_calls(runner), "avg_ms": t_ms,
                                  "algorithmic_bytes": wb, "achieved_gbs": wb / (t_ms * 1e-3) / 1e9}
        if "graph_floor" in bd:
            # the same events around a one-node graph of a one-element add, also after a flush
            kernels["step_writes"]["one_node_graph_floor_ms"] = statistics.median(bd["graph_floor"])
    if "index_topk" in bd:
        t_ms = statistics.mean(bd["index_topk"])
        ib = index_work(wl)
        kernels["index_topk"] = {"launches_per_step": 1, "avg_ms": t_ms, "algorithmic_bytes": ib,
                                 "achieved_gbs": ib / (t_ms * 1e-3) / 1e9}
    if "reindex_topk" in bd:
        t_ms = statistics.mean(bd["reindex_topk"])
        rb = reindex_work(wl)
        kernels["reindex_topk"] = {"launches_per_step": sum(1 for m in runner.modes if m == "I"), "avg_ms": t_ms,
                                   "algorithmic_bytes": rb, "achieved_gbs": rb / (t_ms * 1e-3) / 1e9}
    for k in kernels.values():
        k["hbm_frac"] = k["achieved_gbs"] / hbm_peak
        k["hbm_frac_of_nominal_8tbs"] = k["achieved_gbs"] / 8000.0
    tot = sum(k["avg_ms"] * k["launches_per_step"] for k in kernels.values())
    for k in kernels.values():
        k["share"] = k["avg_ms"] * k["launches_per_step"] / tot if tot else None
    return kernels


def roofline(wl, kernels, peaks):
    """Roofline object of the kernel with the largest share of the step."""
    hbm_peak, tc_peak, _, peak_src = peaks
    if not kernels:
        return None
    dom = max(kernels, key=lambda k: kernels[k]["share"] or 0)
    k = kernels[dom]
    if dom == "sparse_attn":
        traffic, note = attn_traffic(wl.name)
        roof = {"kernel": "csa2_sparse_attn", "bound": "tensor", "achieved": k["achieved_tflops"],
                "peak": tc_peak, "unit": "TFLOP/s", "frac": k["achieved_tflops"] / tc_peak,
                "traffic": traffic, "traffic_source": note,
                "peak_source": f"{peak_src} bf16_tflops (fp16 MMA runs at the same rate)",
                "hbm_achieved_gbs": k["achieved_gbs"], "hbm_frac": k["achieved_gbs"] / hbm_peak,
                "hbm_frac_of_nominal_8tbs": k["achieved_gbs"] / 8000.0}
        if wl.prefill_start is not None:
            roof["note"] = ("prefill: the selected rows are gathered from a cache that stays in L2, "
                            "so the per-query bytes exceed what crosses HBM")
        return roof
    name = {"index_topk": "csa2_index_topk", "reindex_topk": "csa2_index_topk (Reindex)",
            "step_writes": "csa2_quantize_kv_batch"}[dom]
    return {"kernel": name, "bound": "hbm", "achieved": k["achieved_gbs"], "peak": hbm_peak, "unit": "GB/s",
            "frac": k["achieved_gbs"] / hbm_peak, "traffic": None, "traffic_source": "no capture",
            "peak_source": f"{peak_src} hbm_gbs"}


def max_over_ranks(torch, dist, value, world, device="cuda"):
    """The largest of the ranks' values: a multi-GPU time is the slowest rank's.  One rank: the
    value itself, with no collective."""
    if world <= 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(rows_per_rank, world, steps, total_ms):
    """Queries per second of the whole job: every rank's rows for every step, over the slowest
    rank's total time."""
    return rows_per_rank * world * steps / (total_ms / 1e3)


def measure_workload(torch, csa2, args, wl, world, rank, local, peaks, flush, detail=True):
    """Time the workload's step (graph replays, L2 flushed before each) and, with detail, the
    per-call breakdown, roofline, e2e and the oracle's CPU baseline."""
    import torch.distributed as dist
    from compressed_sparse_attention_quantize_b200 import runtime
    runner = runtime.GroupRunner(wl, out_dtype=csa2.DTYPE_BF16)
    # the timed step: the step's quantise-on-write (newest entry and indexer key per sequence,
    # indexer queries, window entries of the step token) in one launch, then the layer group;
    # replayed as one CUDA graph (--eager: one call each per step).  If the writes fail on their
    # first run (an argument the library rejects), the step falls back to the group alone and
    # says so.
    writes = True
    writes_note = STEP_WRITES
    try:
        runner.write_step()
        torch.cuda.synchronize()
    except Exception as exc:
        writes = False
        writes_note = f"not run: {type(exc).__name__}: {exc}"[:300]
    step_fn = runner.step if writes else runner.run
    graph_kernels = 0
    if not args.eager:
        graph_kernels = runner.capture(with_writes=writes)
        step_fn = runner.replay
    for _ in range(args.warmup):
        flush()
        step_fn()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = csa2.csa2_launch_count()
    with ClockSampler(torch.cuda.current_device() if world == 1 else local) as clk:
        ms = time_steps(torch, step_fn, args.steps, flush)
    # graph replays do not pass through the library's launch counter: count the graph's kernels
    launches = csa2.csa2_launch_count() - launches0 + graph_kernels * args.steps
    clocks = clk.summary()
    total_ms = max_over_ranks(torch, dist, sum(ms), world)
    if world > 1:
        dist.barrier()
    rows = wl.B * wl.T
    res = {"value": replica_throughput(rows, world, args.steps, total_ms), "unit": UNIT,
           "ms_per_step": total_ms / args.steps, "steps": args.steps, "warmup": args.warmup,
           "gpu_launches": int(launches), "clocks": clocks,
           "config": {"workload": wl.name, "batch_per_gpu": wl.B, "queries_per_sequence": wl.T,
                      "ctx_tokens": wl.ctx_tokens[0] if len(set(wl.ctx_tokens)) == 1 else wl.ctx_tokens,
                      "entries_per_seq": wl.n_entries[0] if len(set(wl.n_entries)) == 1 else wl.n_entries,
                      "layers": ",".join(wl.modes), "heads": wl.H, "index_heads": wl.HI, "topk": wl.K,
                      "pool": wl.P, "swa": 128, "out": "bf16", "step": "eager" if args.eager else "cuda graph",
                      "step_writes": writes_note,
                      "parallelism": f"replicas x{world} (independent sequences)",
                      "l2": "flushed between steps (256 MB write, outside the events)"}}
    if not detail:
        del runner
        return res
    bd = breakdown(torch, csa2, runner, max(3, min(args.steps, 10)), flush, writes)
    kernels = kernel_table(wl, runner, bd, peaks, 2)
    res["kernels"] = kernels
    res["roofline"] = roofline(wl, kernels, peaks)
    e2e = e2e_measure(torch, csa2, runner, max(3, min(args.steps, 10)), 2, flush, writes)
    if world > 1:
        e2e["ms_per_step"] = max_over_ranks(torch, dist, e2e["ms_per_step"], world)
        e2e["value"] = replica_throughput(rows, world, 1, e2e["ms_per_step"])
    res["e2e"] = e2e
    softmax_scale = runner.softmax_scale
    del runner
    torch.cuda.empty_cache()
    res["cpu_baseline"] = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, softmax_scale, budget_s=15.0 if args.config == wl.seed else 4.0)
    return res


def run_csa2(args, wl):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    import compressed_sparse_attention_quantize_b200 as csa2
    from compressed_sparse_attention_quantize_b200 import build as csa2_build, synth
    if not os.path.exists(csa2.library_path()):
        csa2_build.build()

    def replica(w):
        if rank > 0:
            w.seed = w.seed + 1000 * rank          # independent sequences per rank
        return w

    peaks = _peaks()
    flush_buf = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device="cuda")

    def flush():
        flush_buf.fill_(1)

    head = measure_workload(torch, csa2, args, replica(wl), world, rank, local, peaks, flush,
                            detail=not args.quick)
    if args.quick:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                              "config": {"workload": wl.name}, "gpu_launches": head["gpu_launches"],
                              "clocks": head["clocks"], "quick": True}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    # the other timed workloads (decode at 1M context first: the metric's second context)
    workloads = {}
    if not args.no_workloads and not args.entries:
        for c in (3, 2, 4):
            if c == args.config:
                continue
            w = replica(synth.workload(c))
            try:
                r = measure_workload(torch, csa2, args, w, world, rank, local, peaks, flush)
            except Exception as exc:              # one workload never costs the headline line
                torch.cuda.synchronize()
                r = {"error": f"{type(exc).__name__}: {exc}"[:300]}
            r.pop("steps", None)
            r.pop("warmup", None)
            workloads[w.name] = r

    try:
        side = topk_side_reference(torch, csa2, wl, flush)
    except Exception as exc:                 # a side reference never costs the main line
        side = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None,
                "dtype": "f16 MMA (attention), fp4 MMA (indexer), f32 accumulate",
                "data": "synthetic (seeded; shapes and distributions of the workload)",
                "config": head["config"], "roofline": head["roofline"], "kernels": head["kernels"],
                "cpu_baseline": head["cpu_baseline"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
                "clocks": head["clocks"], "workloads": workloads, "topk_side_reference": side}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["csa2", "reference"], default="csa2")
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time the --config workload only (no 'workloads' object)")
    ap.add_argument("--eager", action="store_true", help="time one csa2_layer_group call per step "
                    "instead of replaying it as a CUDA graph")
    ap.add_argument("--quick", action="store_true",
                    help="timed region only (no breakdown, e2e or CPU baseline): for profiler captures")
    ap.add_argument("--entries", type=int, default=0,
                    help="override compressed entries per sequence (smaller profiling cases)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from compressed_sparse_attention_quantize_b200 import synth
    wl = synth.workload(args.config)
    if args.entries:
        wl = synth.scaled(wl, n=args.entries, name=f"{wl.name}_n{args.entries}")
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_csa2(args, wl)


if __name__ == "__main__":
    main()
