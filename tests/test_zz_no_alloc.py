"""wq_gemm_w4a16_noalloc: the W4A16 entry point for callers that cannot allocate.

Callers such as graph-building runtimes, plug-in hosts that own all device
memory, or fixed-budget deployments cannot call cudaMalloc to provide the
workspace wq_gemm_w4a16 asks for; this entry point takes none and uses the
library's fixed scratch array.  Its results must match the regular entry
point's within the tolerance every matmul test here uses
(|y - y_ref| <= 4e-3 * sum_k |x * w_hat|), on two calls in a row (the second
call finds the array as the first left it), and each call must also meet that
bound against the oracle's binary64 product on its own, so that the two
kernels' errors cannot add up unnoticed.  One shape needs exactly the array's
2 MiB.  This file is collected last, so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import group_wise_weight_b200 as wq
import oracle
import wq_inputs
from group_wise_weight_b200 import build as wqbuild

pytestmark = pytest.mark.gpu
TOL = 4e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    wqbuild.build()
    wq.lib()


def _quantised(N, K, seed):
    w = wq_inputs.llm_weight(N, K, seed)
    q, s, z = wq.wq_quantize_int4(w.cuda(), 128)
    codes, so, zo = oracle.quantize_int4(w.float().numpy(), 128)
    return q, s, z, codes, so, zo


# (16, 32752, 256): M * N * 4 bytes plus one int per 128 rows, each rounded up to 256 bytes, is exactly
# the array's 2 MiB -- the largest N accepted at M = 16 (N = 32753 is refused, tests/test_abi.py).
@pytest.mark.parametrize("M,N,K", [(2, 1000, 512), (8, 14336, 4096), (16, 4096, 8192), (5, 300, 256),
                                   (16, 32752, 256)])
def test_noalloc_matches_regular_entry_point_twice(M, N, K):
    q, s, z, codes, so, zo = _quantised(N, K, 900 + M)
    x = wq_inputs.activations(M, K, 901 + M).cuda()
    y_ref = wq.wq_gemm_w4a16(x, q, s, z, 128)
    torch.cuda.synchronize()
    y_exact, a_ref = oracle.gemm_w4a16(x.double().cpu().numpy(), codes, so, zo, 128)
    bound = TOL * a_ref
    yr = y_ref.double().cpu().numpy()
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        wq.wq_gemm_w4a16_noalloc(x, q, s, z, 128, y=y)
        torch.cuda.synchronize()
        yn = y.double().cpu().numpy()
        assert np.all(np.isfinite(yn)), f"call {call}: output not fully written"
        assert np.all(np.abs(yn - yr) <= bound), f"call {call}: differs from wq_gemm_w4a16"
        assert np.all(np.abs(yn - y_exact) <= bound), f"call {call}: outside the bound against the oracle"
    assert wq.wq_device_status() == wq.WQ_OK


def test_noalloc_rejects_shapes_beyond_its_scratch():
    M, N, K = 16, 57344, 256  # 16 * 57344 * 4 bytes > 2 MiB
    q = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.zeros((N, K // 128), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_gemm_w4a16_noalloc(x, q, s, s, 128)
    assert e.value.status == wq.WQ_ERR_WORKSPACE
    assert "scratch" in wq.wq_last_error()


def test_noalloc_rejects_unsupported_shapes():
    q = torch.zeros((256, 256), dtype=torch.uint8, device="cuda")
    s = torch.zeros((256, 8), dtype=torch.bfloat16, device="cuda")
    for M, g in ((1, 128), (17, 128), (4, 64)):
        x = torch.zeros((M, 512), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(wq.WQError) as e:
            wq.wq_gemm_w4a16_noalloc(x, q, s, s, g)
        assert e.value.status == wq.WQ_ERR_UNSUPPORTED
