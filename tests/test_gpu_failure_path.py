"""The bounded-wait failure path on the GPU, made to happen without a fault.

Every barrier wait in the library's kernels gives up after about a second, records WQ_ERR_DEVICE_TIMEOUT in
the device status word and lets the kernel wind down (its copies in flight drained, its tensor memory
freed).  The test hook wq_test_skip_weight_copy makes the next tensor-core W4A16 launch never request one
weight copy, so the waits on that copy run out.  The call must return, wq_device_status must report the
timeout (and clear it), and after the workspace is zero-filled again, as wq.h requires after a timeout, the
next call must match the oracle.
"""
import time

import numpy as np
import pytest
import torch

import group_wise_weight_b200 as wq
import oracle
import wq_inputs
from group_wise_weight_b200 import build as wqbuild

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    wqbuild.build()
    wq.lib()
    torch.cuda.init()


def test_a_wait_that_runs_out_returns_and_leaves_the_library_usable():
    M, N, K = 128, 1024, 2048
    w = wq_inputs.llm_weight(N, K, 700)
    x = wq_inputs.activations(M, K, 701).cuda()
    q, s, z = wq.wq_quantize_int4(w.cuda(), 128)
    ws = torch.zeros(wq.wq_gemm_workspace_bytes(M, N, K, 128, 4), dtype=torch.uint8, device="cuda")
    assert wq.wq_device_status() == wq.WQ_OK
    wq.lib().wq_test_skip_weight_copy(3)
    t0 = time.perf_counter()
    wq.wq_gemm_w4a16(x, q, s, z, 128, workspace=ws)
    assert wq.wq_device_status() == wq.WQ_ERR_DEVICE_TIMEOUT
    assert time.perf_counter() - t0 < 30.0
    assert wq.wq_device_status() == wq.WQ_OK  # read and cleared
    ws.zero_()
    y = wq.wq_gemm_w4a16(x, q, s, z, 128, workspace=ws)
    torch.cuda.synchronize()
    assert wq.wq_device_status() == wq.WQ_OK
    codes, so, zo = oracle.quantize_int4(w.float().numpy(), 128)
    y_ref, a_ref = oracle.gemm_w4a16(x.double().cpu().numpy(), codes, so, zo, 128)
    err = np.abs(y.double().cpu().numpy() - y_ref)
    assert np.all(err <= 4e-3 * a_ref)
