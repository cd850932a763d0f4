"""FP8 quantisers and the FP8 W8A8 tensor-core matmul against the CPU oracle.

"Quantization for LLM inference: FP8, INT4 (GPTQ, AWQ) and GGUF", section "FP8: the Hopper/Blackwell
datacenter format".  Codes and scales must be bit-exact against oracle.quantize_fp8_rows /
quantize_fp8_tensor; the matmul must satisfy, element by element,
    |y - y_ref| <= 4e-3 * sum_k |x_hat[m][k] * w_hat[n][k]|
against oracle.gemm_w8a8_fp8 (binary64 sums of the decoded values).
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
FMTS = {"e4m3": (wq.WQ_FP8_E4M3, oracle.E4M3), "e5m2": (wq.WQ_FP8_E5M2, oracle.E5M2)}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    wqbuild.build()
    wq.lib()
    torch.cuda.init()


@pytest.fixture(autouse=True)
def _no_device_timeouts():
    yield
    assert wq.wq_device_status() == wq.WQ_OK, "a kernel recorded a bounded-wait timeout"


def check_rows(w: torch.Tensor, fmt: str):
    q, s = wq.wq_quantize_fp8(w.cuda(), FMTS[fmt][0])
    torch.cuda.synchronize()
    codes, so = oracle.quantize_fp8_rows(w.float().numpy(), FMTS[fmt][1])
    assert np.array_equal(q.cpu().numpy(), codes), "FP8 codes differ"
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32)), "scales differ"
    return q, s


def extreme_rows(K: int, seed: int, dtype) -> torch.Tensor:
    """Rows that reach the corners of the format: an all-zero row, subnormal codes next to a large value,
    exact FP8 values (ties after scaling), magnitudes 2^+-100, one-signed rows."""
    g = torch.Generator().manual_seed(seed)
    rows = [torch.zeros(K),
            torch.randn(K, generator=g) * 1e-6,
            torch.randn(K, generator=g) * 2.0 ** 100,
            torch.randn(K, generator=g) * 2.0 ** -100,
            torch.rand(K, generator=g) + 0.5]
    r = torch.randn(K, generator=g) * 1e-4
    r[7] = 448.0
    rows.append(r)  # scale 1: the small values land on FP8 subnormals
    t = torch.randint(-64, 64, (K,), generator=g).float() * 0.5 + 0.25
    t[3] = 448.0
    rows.append(t)  # scale 1: quarter-steps half way between E4M3 values
    return torch.stack(rows).to(dtype)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_fp8_rows(fmt, dtype):
    w = wq_inputs.llm_weight(300, 1024, 31, dtype=dtype)
    check_rows(w, fmt)
    check_rows(extreme_rows(256, 32, dtype), fmt)


def test_quantize_fp8_rows_padded_leading_dimension():
    w = wq_inputs.llm_weight(64, 1024, 33, dtype=torch.bfloat16)
    wp = torch.zeros((64, 1088), dtype=torch.bfloat16)
    wp[:, :1024] = w
    wp[:, 1024:] = 1e4  # never read
    q, s = wq.wq_quantize_fp8(wp.cuda()[:, :1024], wq.WQ_FP8_E4M3)
    torch.cuda.synchronize()
    codes, so = oracle.quantize_fp8_rows(w.float().numpy(), oracle.E4M3)
    assert np.array_equal(q.cpu().numpy(), codes)
    assert np.array_equal(s.cpu().numpy(), so)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M,K", [(1, 4096), (7, 96), (128, 8192)])
def test_quantize_fp8_tensor(fmt, dtype, M, K):
    x = wq_inputs.activations(M, K, 40 + M).to(dtype)
    q, s = wq.wq_quantize_fp8_tensor(x.cuda(), FMTS[fmt][0])
    torch.cuda.synchronize()
    codes, so = oracle.quantize_fp8_tensor(x.float().numpy(), FMTS[fmt][1])
    assert np.array_equal(q.cpu().numpy(), codes), "FP8 codes differ"
    assert s.cpu().numpy()[0].view(np.uint32) == np.float32(so).view(np.uint32), "scale differs"


def test_quantize_fp8_tensor_all_zero_and_repeated_calls():
    x = torch.zeros((3, 64), dtype=torch.bfloat16, device="cuda")
    q, s = wq.wq_quantize_fp8_tensor(x)
    assert float(s.item()) == 1.0 and int(q.abs().sum()) == 0
    # the scale buffer holds the maximum between the kernels of one call: a second call must not see the
    # first call's scale
    y = wq_inputs.activations(4, 256, 5).cuda()
    for _ in range(2):
        q, s = wq.wq_quantize_fp8_tensor(y, scale=s, q=torch.empty((4, 256), dtype=torch.uint8, device="cuda"))
        torch.cuda.synchronize()
        codes, so = oracle.quantize_fp8_tensor(y.float().cpu().numpy(), oracle.E4M3)
        assert np.array_equal(q.cpu().numpy(), codes) and float(s.item()) == float(so)


def gemm_case(M, N, K, seed, wgen=None, rows=None):
    """GPU: both quantisers then the matmul; oracle: gemm_w8a8_fp8 on the same inputs (optionally only the
    given weight rows, quantised per row exactly as in the full matrix)."""
    w = wgen(N, K, seed) if wgen else wq_inputs.llm_weight(N, K, seed, dtype=torch.bfloat16)
    x = wq_inputs.activations(M, K, seed + 1)
    wd, xd = w.cuda(), x.cuda()
    qw, sw = wq.wq_quantize_fp8(wd)
    qx, sx = wq.wq_quantize_fp8_tensor(xd)
    y = wq.wq_gemm_w8a8_fp8(qx, sx, qw, sw)
    torch.cuda.synchronize()
    sel = np.arange(N) if rows is None else rows
    y_ref, a_ref = oracle.gemm_w8a8_fp8(x.float().numpy(), w.float().numpy()[sel])
    yg = y.double().cpu().numpy()[:, sel]
    err = np.abs(yg - y_ref)
    bad = err > TOL * a_ref
    ratio = float(np.max(err / np.where(a_ref > 0, a_ref, 1.0)))
    assert not bad.any(), f"{bad.sum()} outputs outside 4e-3*sum|x*w_hat|; max ratio {ratio:.3e}"
    return y, (qx, sx, qw, sw)


@pytest.mark.parametrize("M", [1, 2, 16, 31, 32, 33, 64, 100, 128, 129, 256, 300])
def test_gemm_w8a8_fp8_batch_sizes(M):
    gemm_case(M, 384, 1024, 50 + M)


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (17, 129, 256), (128, 1000, 2048), (64, 4096, 4096),
                                   (256, 200, 8192), (8, 10240, 1024)])
def test_gemm_w8a8_fp8_shapes(M, N, K):
    gemm_case(M, N, K, 70 + M + N % 97)


def test_gemm_w8a8_fp8_full70b_gate_up_sampled():
    N, K = 57344, 8192
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(N, 48, replace=False), [0, N - 1]]))
    gemm_case(128, N, K, 90, rows=rows)


def test_gemm_w8a8_fp8_repeatable_and_zero_rows():
    M, N, K = 128, 2048, 8192  # K-split tiles: per-segment partials summed in a fixed order
    w = wq_inputs.llm_weight(N, K, 91, dtype=torch.bfloat16)
    w[5] = 0
    x = wq_inputs.activations(M, K, 92).cuda()
    qw, sw = wq.wq_quantize_fp8(w.cuda())
    qx, sx = wq.wq_quantize_fp8_tensor(x)
    ws = torch.zeros(wq.wq_gemm_w8a8_fp8_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    y1 = wq.wq_gemm_w8a8_fp8(qx, sx, qw, sw, workspace=ws)
    y2 = wq.wq_gemm_w8a8_fp8(qx, sx, qw, sw, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert int(y1[:, 5].float().abs().sum()) == 0


def test_gemm_w8a8_fp8_rejects_bad_arguments():
    q = torch.zeros((256, 192), dtype=torch.uint8, device="cuda")
    s = torch.ones(256, dtype=torch.float32, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_gemm_w8a8_fp8(q[:4], s[:1], q, s)  # K = 192
    assert e.value.status == wq.WQ_ERR_SHAPE
