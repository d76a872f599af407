"""Failure detection on the GPU without a fault: a bounded device wait that runs out.

The self-test kernel's producer skips its mbarrier arrival on the host's instruction.  The
consumer's bounded wait (the one the pipelined kernels use) gives up, records
CSA2_ERR_TIMEOUT in the device error word, and the kernel exits.  The test checks that
status, that reading the word clears it, and that the same context then runs a
parity-checked call.
"""
import numpy as np
import pytest
import torch

import oracle
import compressed_sparse_attention_quantize_b200 as csa2
from compressed_sparse_attention_quantize_b200 import runtime

pytestmark = pytest.mark.gpu

CSA2_ERR_TIMEOUT = 6


def test_bounded_wait_timeout_is_reported_and_context_survives():
    assert csa2.csa2_device_error() == 0
    csa2.csa2_selftest_bounded_wait(False)              # handshake completes
    assert csa2.csa2_device_error() == 0
    csa2.csa2_selftest_bounded_wait(True)               # the arrival never comes
    assert csa2.csa2_device_error() == CSA2_ERR_TIMEOUT
    assert csa2.csa2_device_error() == 0                # read-and-clear
    csa2.csa2_selftest_bounded_wait(True)
    csa2.csa2_selftest_bounded_wait(False)              # a later good run does not hide it
    assert csa2.csa2_device_error() == CSA2_ERR_TIMEOUT

    x = np.random.default_rng(7).standard_normal((64, 512)).astype(np.float32)
    rows = torch.zeros((64, 288), dtype=torch.uint8, device="cuda")
    runtime.quantize_fp4_rows(torch.from_numpy(x).cuda(), rows, rows[:, 256:], 288, 288)
    torch.cuda.synchronize()
    oc, os_ = oracle.quantize_fp4(x)
    got = rows.cpu().numpy()
    assert np.array_equal(got[:, :256], oc) and np.array_equal(got[:, 256:], os_)
    assert csa2.csa2_device_error() == 0
