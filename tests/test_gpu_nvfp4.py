"""NVFP4 quantiser and the NVFP4 W4A4 block-scaled tensor-core matmul against the CPU oracle.

"Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache Quantization", section "Hardware,
formats and the roofline" (E2M1 values, an E4M3 scale per 16 values, a binary32 tensor scale).  Codes,
block scales and tensor scales must be bit-exact against oracle.quantize_nvfp4 (the block scales after
undoing the library's tensor-core layout); the matmul must satisfy, element by element,
    |y - y_ref| <= 4e-3 * sum_k |x_hat[m][k] * w_hat[n][k]|
against oracle.gemm_nvfp4 (binary64 sums of the decoded values).
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
    torch.cuda.init()


@pytest.fixture(autouse=True)
def _no_device_timeouts():
    yield
    assert wq.wq_device_status() == wq.WQ_OK, "a kernel recorded a bounded-wait timeout"


def scales_as_rows(sf: np.ndarray, N: int, K: int) -> np.ndarray:
    """[N][K/16] block scales from the tensor-core layout: the scale of (row r, block b) sits at byte
    16 (r % 32) + 4 ((r % 128) / 32) + (b % 4) of the 512-byte atom (r / 128) * (K / 64) + b / 4."""
    r = np.arange(N)[:, None]
    b = np.arange(K // 16)[None, :]
    off = ((r // 128) * (K // 64) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)
    return sf[off]


def check_quant(w: torch.Tensor, wd: torch.Tensor = None):
    wd = w.cuda() if wd is None else wd
    N, K = w.shape
    c, sf, ts = wq.wq_quantize_nvfp4(wd)
    torch.cuda.synchronize()
    codes, blocks, st = oracle.quantize_nvfp4(w.float().numpy())
    assert np.array_equal(c.cpu().numpy(), oracle.pack_int4(codes)), "E2M1 codes differ"
    sfh = sf.cpu().numpy()
    assert np.array_equal(scales_as_rows(sfh, N, K), blocks), "block scales differ"
    pad = np.ones(sfh.size, dtype=bool)
    r = np.arange(N)[:, None]
    b = np.arange(K // 16)[None, :]
    pad[(((r // 128) * (K // 64) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)).ravel()] = False
    assert not sfh[pad].any(), "padding rows of the block scales are not zero"
    assert ts.cpu().numpy()[0].view(np.uint32) == np.float32(st).view(np.uint32), "tensor scale differs"
    return c, sf, ts


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,K", [(128, 64), (300, 1024), (64, 8192)])
def test_quantize_nvfp4(dtype, N, K):
    check_quant(wq_inputs.llm_weight(N, K, 100 + N, dtype=dtype))


def test_quantize_nvfp4_special_blocks():
    """An all-zero block, a block whose scale rounds to 0 (codes 0), blocks of exact E2M1 values and ties,
    negative values that round to -0, and one outlier setting the tensor scale."""
    g = torch.Generator().manual_seed(7)
    w = torch.randn(130, 256, generator=g) * 0.02
    w[0, :16] = 0.0
    w[1, 16:32] = 1e-7
    w[2, :16] = torch.tensor([0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -0.5, 5.0]) * 0.01
    w[3, :16] = -1e-4
    w[4, :16] = -1e-5
    w[4, 0] = 0.01  # the small negatives round to -0 (code 8)
    w[129, 200] = 3.0
    check_quant(w)
    check_quant(torch.zeros(5, 128))


def test_quantize_nvfp4_padded_rows():
    w = wq_inputs.llm_weight(40, 512, 8, dtype=torch.bfloat16)
    wp = torch.full((40, 576), 100.0, dtype=torch.bfloat16)
    wp[:, :512] = w
    check_quant(w, wp.cuda()[:, :512])


def gemm_case(M, N, K, seed, rows=None):
    w = wq_inputs.llm_weight(N, K, seed, dtype=torch.bfloat16)
    x = wq_inputs.activations(M, K, seed + 1)
    xc, xsf, xts = wq.wq_quantize_nvfp4(x.cuda())
    wc, wsf, wts = wq.wq_quantize_nvfp4(w.cuda())
    y = wq.wq_gemm_nvfp4(xc, xsf, xts, wc, wsf, wts)
    torch.cuda.synchronize()
    wf = w.float().numpy()
    if rows is None:
        sel = np.arange(N)
        y_ref, a_ref = oracle.gemm_nvfp4(x.float().numpy(), wf)
    else:
        # the tensor scale depends only on the largest magnitude: quantising the sampled rows together
        # with the row that holds it reproduces the full matrix's codes for those rows
        top = int(np.argmax(np.abs(wf).max(axis=1)))
        sel = np.unique(np.concatenate([rows, [top]]))
        y_ref, a_ref = oracle.gemm_nvfp4(x.float().numpy(), wf[sel])
    yg = y.double().cpu().numpy()[:, sel]
    err = np.abs(yg - y_ref)
    bad = err > TOL * a_ref
    ratio = float(np.max(err / np.where(a_ref > 0, a_ref, 1.0)))
    assert not bad.any(), f"{bad.sum()} outputs outside 4e-3*sum|x*w_hat|; max ratio {ratio:.3e}"
    return y


@pytest.mark.parametrize("M", [1, 2, 17, 100, 128, 129, 256])
def test_gemm_nvfp4_batch_sizes(M):
    gemm_case(M, 384, 1024, 120 + M)


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (128, 1000, 2048), (64, 4096, 4096), (128, 200, 8192)])
def test_gemm_nvfp4_shapes(M, N, K):
    gemm_case(M, N, K, 140 + N % 89)


def test_gemm_nvfp4_full70b_gate_up_sampled():
    N, K = 57344, 8192
    rows = np.random.default_rng(4).choice(N, 48, replace=False)
    gemm_case(128, N, K, 150, rows=np.concatenate([rows, [0, N - 1]]))


def test_gemm_nvfp4_repeatable():
    M, N, K = 128, 2048, 8192
    w = wq_inputs.llm_weight(N, K, 160, dtype=torch.bfloat16).cuda()
    x = wq_inputs.activations(M, K, 161).cuda()
    xq = wq.wq_quantize_nvfp4(x)
    wqq = wq.wq_quantize_nvfp4(w)
    ws = torch.zeros(wq.wq_gemm_nvfp4_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    y1 = wq.wq_gemm_nvfp4(*xq, *wqq, workspace=ws)
    y2 = wq.wq_gemm_nvfp4(*xq, *wqq, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
