"""The end-to-end step as the benchmark runs it -- host inputs in csa2_host_alloc buffers, staged
copies and quantise-on-write on a second stream, each layer waiting on its own ready events, the
step captured as one CUDA graph -- leaves the same outputs as the step run from device inputs."""
import pytest
import torch

import bench
import compressed_sparse_attention_quantize_b200 as csa2
from compressed_sparse_attention_quantize_b200 import runtime, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("config,kw", [(1, dict(B=4, n=8192, K=512)),
                                       (2, dict(B=4, n=8192, K=512, P=2000))])
def test_e2e_step_matches_device_step(config, kw):
    wl = synth.scaled(synth.workload(config), **kw)
    runner = runtime.GroupRunner(wl, out_dtype=csa2.DTYPE_BF16)
    runner.write_step()
    runner.run()
    torch.cuda.synchronize()
    ref = [ld["out"].clone() for ld in runner.layer_data]
    for ld in runner.layer_data:
        ld["out"].fill_(float("nan"))
    buf = torch.empty((16 << 20,), dtype=torch.uint8, device="cuda")
    r = bench.e2e_measure(torch, csa2, runner, 3, 1, lambda: buf.fill_(1), writes=True)
    torch.cuda.synchronize()
    assert r["h2d_bytes_per_step"] > 0 and r["d2h_bytes_per_step"] > 0
    for l, (a, ld) in enumerate(zip(ref, runner.layer_data)):
        assert torch.equal(a, ld["out"]), l
    # the layer descriptors point at the runner's own buffers again
    for L, ld in zip(runner.layer_descs, runner.layer_data):
        assert L.q == ld["q"].data_ptr()
        if "iw" in ld:
            assert L.iw == ld["iw"].data_ptr()
