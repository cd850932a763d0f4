"""One workspace shared by calls of different shapes and kernels (GPU).

The matmul kernels keep per-tile arrival counters and binary32 partial sums of split tiles in the caller's
workspace, and `include/wq.h` lets a zero-filled workspace serve later calls of any shape on the same stream.
A call re-zeroes its counters but leaves its partial sums behind, so that holds only if no later call can
find its counters on an earlier call's partial sums (its split tiles would then never be combined): every
kernel keeps its counters in the first 64 KB and its partial sums above.  Each call below runs on one shared
workspace sized for the largest of them; after each, the counter region must be zero again and y must equal,
bit for bit, the same call on a fresh workspace.  The calls with the largest partial-sum regions come first.
"""
COUNTER_REGION = 65536
import pytest
import torch

import group_wise_weight_b200 as wq
import wq_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    wq.lib()
    yield


def _w4(N, K, g, seed, dev):
    return wq.wq_quantize_int4(wq_inputs.llm_weight(N, K, seed, device=dev), g)


def _calls(dev):
    """(name, fn(workspace) -> y, workspace bytes, bit-reproducible)."""
    calls = []

    def w4(name, M, N, K, g, seed):
        q, s, z = _w4(N, K, g, seed, dev)
        x = wq_inputs.activations(M, K, seed + 1, device=dev)
        calls.append((name, lambda ws: wq.wq_gemm_w4a16(x, q, s, z, g, workspace=ws),
                      wq.wq_gemm_workspace_bytes(M, N, K, g, 4), not (2 <= M <= 16 and K % 1024 != 0)))

    def w8(name, M, N, K, seed):
        q8, s8 = wq.wq_quantize_int8(wq_inputs.llm_weight(N, K, seed, device=dev), None)
        x = wq_inputs.activations(M, K, seed + 1, device=dev)
        calls.append((name, lambda ws: wq.wq_gemm_w8a16(x, q8, s8, None, workspace=ws),
                      wq.wq_gemm_workspace_bytes(M, N, K, K, 8), True))

    w4("w4a16 M=128 g128 (128 x 128 tiles)", 128, 4096, 8192, 128, 11)
    w4("w4a16 M=1 g128 gate+up-like", 1, 20000, 8192, 128, 13)
    w4("w4a16 M=1 g128 long K", 1, 8192, 28672, 128, 15)
    w4("w4a16 M=1 g32", 1, 3000, 4096, 32, 17)
    w4("w4a16 M=2 (integer small batch)", 2, 3000, 4096, 128, 19)
    w4("w4a16 M=8 (bf16 small batch)", 8, 3000, 4096, 128, 21)
    w4("w4a16 M=16 (128 x 128 tiles)", 16, 4097, 2048, 128, 23)
    w4("w4a16 M=40 g64 (combined tensor-core kernel)", 40, 384, 2048, 64, 25)
    w4("w4a16 M=4 K=1152 (TMA kernel, atomics)", 4, 1000, 1152, 128, 27)
    w8("w8a16 M=1 per channel (integer kernel)", 1, 8192, 8192, 29)
    w8("w8a16 M=128 per channel (tensor cores)", 128, 1024, 4096, 31)

    # column-scaled at M = 8: the scaled activations are staged at the front of the workspace
    N, K = 2048, 4096
    cs = wq_inputs.channel_scales(K, 33).to(dev)
    qc, sc_, zc = wq.wq_quantize_int4_scaled(wq_inputs.llm_weight(N, K, 33, dtype=torch.bfloat16, device=dev), cs, 128)
    xc = wq_inputs.activations(8, K, 34, device=dev)
    calls.append(("w4a16 col-scaled M=8", lambda ws: wq.wq_gemm_w4a16_colscaled(xc, cs, qc, sc_, zc, 128, workspace=ws),
                  int(wq.lib().wq_gemm_w4a16_colscaled_workspace_bytes(8, N, K, 128)), True))

    # FP8 W8A8 and NVFP4 W4A4 at M = 128
    N, K = 1024, 4096
    wf = wq_inputs.llm_weight(N, K, 35, device=dev)
    xf = wq_inputs.activations(128, K, 36, device=dev)
    qw, sw = wq.wq_quantize_fp8(wf)
    qx, sx = wq.wq_quantize_fp8_tensor(xf)
    calls.append(("fp8 W8A8 M=128", lambda ws: wq.wq_gemm_w8a8_fp8(qx, sx, qw, sw, workspace=ws),
                  wq.wq_gemm_w8a8_fp8_workspace_bytes(128, N, K), True))
    nw, nx = wq.wq_quantize_nvfp4(wf), wq.wq_quantize_nvfp4(xf)
    calls.append(("nvfp4 W4A4 M=128", lambda ws: wq.wq_gemm_nvfp4(*nx, *nw, workspace=ws),
                  wq.wq_gemm_nvfp4_workspace_bytes(128, N, K), True))
    return calls


def test_one_workspace_serves_every_shape_and_kernel():
    dev = torch.device("cuda", 0)
    calls = _calls(dev)
    need = max(n for _, _, n, _ in calls)
    shared = torch.zeros(need + 256, dtype=torch.uint8, device=dev)
    for rep in range(2):
        for name, fn, n, exact in calls:
            y = fn(shared).clone()
            torch.cuda.synchronize()
            assert wq.wq_device_status() == wq.WQ_OK, name
            left = int(torch.count_nonzero(shared[:COUNTER_REGION]).item())
            assert left == 0, f"{name} (pass {rep}) left {left} non-zero bytes in the counter region"
            fresh = torch.zeros(max(n, 16), dtype=torch.uint8, device=dev)
            y2 = fn(fresh)
            torch.cuda.synchronize()
            if exact:
                assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), f"{name} (pass {rep}): y differs"
            else:
                assert torch.allclose(y.float(), y2.float(), rtol=1e-2, atol=1e-2), f"{name} (pass {rep}): y differs"


def test_more_than_16384_tiles_after_a_smaller_shape():
    """A shape of more than 16,384 tiles keeps counters above 64 KB, where an earlier call's partial sums lie:
    the library clears them before its launch.  M = 1, N = 4,325,376 (16,896 tiles of 256 rows), K = 1024,
    with random codes, scales and zero-points (no quantiser pass over a 8.6 GB weight), after a smaller M = 1
    call on the same workspace; y must equal the same call on a fresh workspace bit for bit."""
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(4242)
    ntiles = 16896
    N, K = 256 * ntiles, 1024
    q = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
    s = (0.001 + 0.01 * torch.rand((N, K // 128), device=dev, generator=g)).to(torch.bfloat16)
    z = torch.randint(0, 16, (N, K // 128), device=dev, generator=g).to(torch.bfloat16)
    x = wq_inputs.activations(1, K, 4243, device=dev)
    need = wq.wq_gemm_workspace_bytes(1, N, K, 128, 4)
    assert need > 2 * COUNTER_REGION  # the counter region reaches past 64 KB
    qs, ss, zs = _w4(20000, 8192, 128, 4244, dev)
    xs = wq_inputs.activations(1, 8192, 4245, device=dev)
    small_need = wq.wq_gemm_workspace_bytes(1, 20000, 8192, 128, 4)
    shared = torch.zeros(max(need, small_need) + 256, dtype=torch.uint8, device=dev)
    wq.wq_gemm_w4a16(xs, qs, ss, zs, 128, workspace=shared)  # leaves partial sums above 64 KB
    torch.cuda.synchronize()
    # the big call's counters beyond 64 KB lie on the smaller call's partial sums
    assert int(torch.count_nonzero(shared[COUNTER_REGION:ntiles * 4]).item()) > 0
    y = wq.wq_gemm_w4a16(x, q, s, z, 128, workspace=shared)
    torch.cuda.synchronize()
    assert wq.wq_device_status() == wq.WQ_OK
    fresh = torch.zeros(need, dtype=torch.uint8, device=dev)
    y2 = wq.wq_gemm_w4a16(x, q, s, z, 128, workspace=fresh)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
