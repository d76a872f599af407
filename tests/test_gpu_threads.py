"""First calls of the library from several host threads at once (GPU, fresh process).

The library sets its per-device launch settings (kernels' shared-memory limits, SM counts,
residency) on first use, under a lock, and the layer group keeps a side stream per host thread.
Here, in a process whose only earlier library calls are the caches' quantise-on-write, four
threads start together on two streams: two run csa2_index_topk + csa2_sparse_attn, two run
csa2_layer_group on runners of their own.  Every result must equal, bit for bit, the same call
made again from one thread afterwards.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import threading
import torch
import compressed_sparse_attention_quantize_b200 as csa2
from compressed_sparse_attention_quantize_b200 import runtime, synth

wl = synth.scaled(synth.workload(1), B=4, n=[3000, 5000, 1000, 4000], K=256, name="threads")
runners = [runtime.GroupRunner(wl, layers=2) for _ in range(3)]
torch.cuda.synchronize()
r = runners[2]
rows = r.rows
streams = [torch.cuda.Stream(), torch.cuda.Stream()]
iws = csa2.csa2_index_topk_workspace_size(0, rows, r.max_n, wl.K, 0)
aws = csa2.csa2_sparse_attn_workspace_size(rows, wl.H, wl.K)
bufs = []
for t in range(2):
    bufs.append(dict(idx=torch.empty((rows, wl.K), dtype=torch.int32, device="cuda"),
                     cnt=torch.empty((rows,), dtype=torch.int32, device="cuda"),
                     out=torch.empty((rows, wl.H, 512), dtype=torch.float32, device="cuda"),
                     iws=torch.empty((iws,), dtype=torch.uint8, device="cuda"),
                     aws=torch.empty((aws,), dtype=torch.uint8, device="cuda")))


def index_attn(t, stream):
    b, ld0, ld = bufs[t], r.layer_data[0], r.layer_data[t]
    csa2.csa2_index_topk(0, ld0["iq_codes"], ld0["iq_scales"], ld0["iw"], wl.B, wl.T, wl.HI, r.k_codes, 32,
                         r.k_scales, 4, r.seq_start, r.n_entries, r.max_n, None, None, None, 0, wl.K, b["idx"],
                         b["cnt"], 0, None, None, b["iws"], iws, stream=stream)
    csa2.csa2_sparse_attn(ld["q"], wl.B, wl.T, wl.H, 512, r.kv, 288, r.seq_start, r.n_entries, b["idx"],
                          b["cnt"], wl.K, ld["swa_codes"], ld["swa_scale"], r.swa_cap, r.swa_start, r.swa_len,
                          r.softmax_scale, b["out"], csa2.DTYPE_F32, None, b["aws"], aws, stream=stream)


errors = []
start = threading.Barrier(4)


def worker(t):
    try:
        s = streams[t % 2]
        start.wait()
        with torch.cuda.stream(s):
            if t < 2:
                index_attn(t, s.cuda_stream)
            else:
                runners[t - 2].run(s.cuda_stream)
        s.synchronize()
    except Exception as exc:
        errors.append(f"thread {t}: {type(exc).__name__}: {exc}")


threads = [threading.Thread(target=worker, args=(t,)) for t in range(4)]
for th in threads:
    th.start()
for th in threads:
    th.join()
torch.cuda.synchronize()
assert not errors, errors
got = [b["out"].clone() for b in bufs] + [[ld["out"].clone() for ld in runners[i].layer_data] for i in range(2)]
got_idx = [b["idx"].clone() for b in bufs]
# the same calls again from this thread
for t in range(2):
    index_attn(t, torch.cuda.current_stream().cuda_stream)
r.run()
torch.cuda.synchronize()
for t in range(2):
    assert torch.equal(got_idx[t], bufs[t]["idx"]), t
    assert torch.equal(got[t], bufs[t]["out"]), t
for i in range(2):
    for l, ld in enumerate(r.layer_data):
        assert torch.equal(got[2 + i][l], ld["out"]), (i, l)
assert csa2.csa2_device_error() == 0
print("THREADS OK")
'''


def test_first_calls_from_four_threads_two_streams():
    env = dict(os.environ)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    p = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert p.returncode == 0 and "THREADS OK" in p.stdout, p.stdout[-2000:] + p.stderr[-4000:]
