"""The activation side of AWQ-style per-input-channel scaling on the GPU against the oracle (oracle/awq.py).

"Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache Quantization", section "The methods
compared" (AWQ scales salient channels; the activations compensate).  wq_gemm_w4a16_colscaled computes
sum_k bf16(x / s) w_hat' with w_hat' the weights w * s quantised by wq_quantize_int4_scaled; the oracle's
compensated product is sum_k (x / s) w_hat' in binary64.  Rounding x / s to bf16 moves each term by at
most 2^-8 of itself and rounding y moves y by at most 2^-8 of |y|; on these inputs the realised error stays
far inside
    |y - y_ref| <= 4e-3 * sum_k |(x / s) w_hat'|
element by element (the bound the matmul tests use; the worst case of the two roundings is 2^-7).  The channel statistics of the search must match the oracle's (magnitudes bit
for bit, scales to the last bit of binary32 up to one unit), and the search through the library's kernels
must pick the oracle pipeline's alpha with the same roundings.
"""
import numpy as np
import pytest
import torch

import group_wise_weight_b200 as wq
import oracle
import wq_inputs
from group_wise_weight_b200 import build as wqbuild
from oracle import awq as oawq

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


@pytest.mark.parametrize("M,N,K,g", [(1, 14336, 4096, 128), (8, 2048, 4096, 128), (128, 1024, 8192, 128),
                                     (1, 300, 512, 64), (40, 256, 1024, 32), (1, 3000, 2048, 32),
                                     (1, 2048, 4096, 64)])
def test_gemm_w4a16_colscaled(M, N, K, g):
    w = wq_inputs.llm_weight(N, K, 300 + M, dtype=torch.bfloat16)
    x = wq_inputs.activations(M, K, 301 + M)
    s = wq_inputs.channel_scales(K, 302 + M)
    q, sc, z = wq.wq_quantize_int4_scaled(w.cuda(), s.cuda(), g)
    y = wq.wq_gemm_w4a16_colscaled(x.cuda(), s.cuda(), q, sc, z, g)
    torch.cuda.synchronize()
    codes, so, zo = oracle.quantize_int4(oawq.scaled_weights(w.float().numpy(), s.numpy()), g)
    assert np.array_equal(q.cpu().numpy(), oracle.pack_int4(codes)), "weight side differs"
    w_hat = oracle.dequant_int4(codes, so, zo, g)
    xs = x.double().numpy() / s.double().numpy()[None, :]
    y_ref = oawq.quantised_product(x.double().numpy(), w_hat, s.numpy())
    _, a_ref = oracle.matmul(xs, w_hat)
    err = np.abs(y.double().cpu().numpy() - y_ref)
    bad = err > TOL * a_ref
    assert not bad.any(), f"{bad.sum()} outputs outside the bound; max ratio {np.max(err / a_ref):.3e}"


@pytest.mark.parametrize("g", [128, 32])
def test_colscaled_m1_matches_prescaled_activations(g):
    """At M = 1 the decode kernel divides x while staging it; the result must equal, bit for bit, the plain
    matmul of bf16(x / s) computed by the pre-pass used at other shapes."""
    N, K = 8192, 8192
    w = wq_inputs.llm_weight(N, K, 310, dtype=torch.bfloat16).cuda()
    s = wq_inputs.channel_scales(K, 311).cuda()
    q, sc, z = wq.wq_quantize_int4_scaled(w, s, g)
    x = wq_inputs.activations(2, K, 312).cuda()
    y1 = wq.wq_gemm_w4a16_colscaled(x[:1], s, q, sc, z, g)     # fused (M = 1 kernel)
    y2 = wq.wq_gemm_w4a16_colscaled(x, s, q, sc, z, g)         # pre-pass, then an M = 2 kernel
    xs = (x[:1].float() / s[None, :]).to(torch.bfloat16)        # torch's IEEE binary32 quotient, RNE to bf16
    y3 = wq.wq_gemm_w4a16(xs, q, sc, z, g)                      # plain M = 1 kernel on pre-scaled x
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y3.view(torch.int16))
    assert np.allclose(y1.float().cpu().numpy(), y2[:1].float().cpu().numpy(), rtol=1e-2, atol=1e-3)


def test_awq_channel_statistics_match_the_oracle():
    x = wq_inputs.activations(48, 1024, 320, channel_seed=321)
    x[:, 7] = 0  # a silent channel takes the smallest positive magnitude
    mag = wq.wq_awq_channel_magnitudes(x.cuda())
    torch.cuda.synchronize()
    m_ref = oawq.channel_magnitude(x.double().numpy())
    assert np.array_equal(mag.cpu().numpy(), m_ref)
    for a in (0.0, 0.05, 0.5, 0.85, 1.0):
        s = wq.wq_awq_channel_scales(mag, a).cpu().numpy()
        s_ref = oawq.channel_scales(m_ref, a)
        ulps = np.abs(s.view(np.int32).astype(np.int64) - s_ref.view(np.int32).astype(np.int64))
        assert ulps.max() <= 1, f"alpha {a}: scales differ by {ulps.max()} ulp"


def test_awq_search_on_the_gpu_tracks_the_oracle_pipeline():
    """The offline search through the library's kernels against the same search run with the oracle's
    quantiser and binary64 matmul on the same roundings (bf16(x / s) with a binary32 quotient, y rounded
    to bf16): the per-alpha errors agree closely and the chosen alpha is the same.  Also against the
    oracle's own binary64 search: its best alpha's error is within 5 % of the oracle's minimum."""
    from group_wise_weight_b200 import awq as gawq
    w = wq_inputs.llm_weight(256, 1024, 411, dtype=torch.float32)
    x = wq_inputs.activations(48, 1024, 412, channel_seed=411)
    alpha, s, errors = gawq.search(w.cuda(), x, 128)
    torch.cuda.synchronize()

    x64 = x.double().numpy()
    exact = x64 @ w.double().numpy().T
    mag = oawq.channel_magnitude(x64)
    ref_errors = []
    for a in gawq.GRID:
        sa = oawq.channel_scales(mag, a)
        codes, so, zo = oracle.quantize_int4(oawq.scaled_weights(w.numpy(), sa), 128)
        xs = (x.float().numpy() / sa[None, :]).astype(np.float32)
        xs = oracle.bf16_value(oracle.bf16_bits(xs)).astype(np.float64)
        y, _ = oracle.gemm_w4a16(xs, codes, so, zo, 128)
        y = oracle.bf16_value(oracle.bf16_bits(y.astype(np.float32))).astype(np.float64)
        ref_errors.append(float(np.sum((y - exact) ** 2)))
    assert np.allclose(errors, ref_errors, rtol=1e-3), np.max(np.abs(np.array(errors) / ref_errors - 1))
    assert gawq.GRID[int(np.argmin(ref_errors))] == alpha

    def deq(w32):
        codes, so, zo = oracle.quantize_int4(w32, 128)
        return oracle.dequant_int4(codes, so, zo, 128)
    _, _, o_errors = oawq.search(x64, w.numpy(), deq)
    assert alpha > 0 and o_errors[gawq.GRID.index(alpha)] <= 1.05 * min(o_errors)
