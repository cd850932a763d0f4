"""Decode attention over an int4 or fp8 KV cache against the CPU oracle (oracle/kv_cache.py).

"Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache Quantization", section "Hardware,
formats and the roofline" (every decode step reads the whole cache); "Quantization for LLM inference: FP8,
INT4 (GPTQ, AWQ) and GGUF", section "KV cache quantization" (fp8 caches; int4 caches in blocks of 128).
The caches are quantised on the GPU by the library's quantisers and must match the oracle's codes and
scales bit for bit; the read must satisfy, element by element,
    |o - o_ref| <= 4e-3 * sum_t p_t |v_hat_t|
with o_ref and the sum from oracle.kv_cache.decode_attention in binary64.  The bound covers the rounding
of p times the token's V scale to the MMA's bf16 (at most 2^-8 = 3.9e-3 of each term; the output stays
binary32) and the binary32 scores and sums.
"""
import numpy as np
import pytest
import torch

import group_wise_weight_b200 as wq
import oracle
import oracle.kv_cache as kv
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


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def quant_int4_gpu(cache: torch.Tensor):
    """The int4 cache format is wq_quantize_int4 with g = 128 on the cache viewed as [B*T*H][D] rows."""
    B, T, H, D = cache.shape
    q, s, z = wq.wq_quantize_int4(cache.cuda().reshape(B * T * H, D), 128)
    return q.reshape(B, T, H, D // 2), s.reshape(B, T, H), z.reshape(B, T, H)


def check_int4_cache(cache, q, s, z):
    codes, so, zo = kv.quantize_kv_int4(cache.float().numpy())
    B, T, H, D = cache.shape
    assert np.array_equal(q.cpu().numpy().reshape(-1, D // 2), oracle.pack_int4(codes.reshape(-1, D)))
    assert np.array_equal(bits(s).ravel(), oracle.bf16_bits(so).ravel())
    assert np.array_equal(bits(z).ravel(), oracle.bf16_bits(zo).ravel())
    return codes, so, zo


def check_o(o: torch.Tensor, o_ref, a_ref):
    og = o.double().cpu().numpy()
    err = np.abs(og - o_ref)
    bad = err > TOL * a_ref
    ratio = float(np.max(err / np.where(a_ref > 0, a_ref, 1.0)))
    assert not bad.any(), f"{bad.sum()} outputs outside 4e-3*sum p|v|; max ratio {ratio:.3e}"
    return ratio


def int4_case(B, T, H, Hq, lengths, seed, offset=0.0):
    kc = wq_inputs.kv_cache(B, T, H, 128, seed, offset)
    vc = wq_inputs.kv_cache(B, T, H, 128, seed + 1, offset)
    qy = wq_inputs.queries(B, Hq, 128, seed + 2)
    kq, ks, kz = quant_int4_gpu(kc)
    vq, vs, vz = quant_int4_gpu(vc)
    lens = torch.tensor(lengths, dtype=torch.int32)
    o = wq.wq_decode_attention_int4(qy.cuda(), kq, ks, kz, vq, vs, vz, lens.cuda())
    torch.cuda.synchronize()
    k_codes, k_s, k_z = check_int4_cache(kc, kq, ks, kz)
    v_codes, v_s, v_z = check_int4_cache(vc, vq, vs, vz)
    o_ref, a_ref = kv.decode_attention(qy.float().numpy(), kv.dequant_kv_int4(k_codes, k_s, k_z),
                                       kv.dequant_kv_int4(v_codes, v_s, v_z), lengths)
    check_o(o, o_ref, a_ref)
    return o


@pytest.mark.parametrize("H,Hq", [(2, 16), (4, 4), (1, 4), (3, 6)])
def test_attention_int4_heads(H, Hq):
    int4_case(3, 700, H, Hq, [0, 700, 333], 10 + H + Hq)


def test_attention_int4_chunk_edges():
    # lengths at and around the 512-token chunk boundary, a single token, and the full cache
    int4_case(6, 1030, 2, 16, [1, 511, 512, 513, 1024, 1030], 30)


def test_attention_int4_far_zero_points():
    # every vector on one side of zero: zero-points far outside [0, 15] for keys and values
    int4_case(2, 300, 2, 8, [300, 77], 40, offset=12.0)


def test_attention_int4_repeatable():
    o1 = int4_case(2, 600, 2, 16, [600, 450], 50)
    o2 = int4_case(2, 600, 2, 16, [600, 450], 50)
    assert torch.equal(o1, o2)


def test_attention_int4_70b_geometry_sampled_batch():
    """The pages' geometry (8 KV heads, 64 query heads, head_dim 128, 8,000-token contexts) on 12 sequences
    with mixed lengths."""
    g = wq_inputs.KV_70B
    B, T = 12, g["T"]
    lengths = [int(x) for x in wq_inputs.sequence_lengths(B, T, 60)]
    lengths[0] = T
    int4_case(B, T, g["H"], g["Hq"], lengths, 61)


def fp8_case(B, T, H, Hq, lengths, seed):
    kc = wq_inputs.kv_cache(B, T, H, 128, seed)
    vc = wq_inputs.kv_cache(B, T, H, 128, seed + 1)
    qy = wq_inputs.queries(B, Hq, 128, seed + 2)
    kq, ks = wq.wq_quantize_fp8_tensor(kc.cuda().reshape(B * T * H, 128))
    vq, vs = wq.wq_quantize_fp8_tensor(vc.cuda().reshape(B * T * H, 128))
    lens = torch.tensor(lengths, dtype=torch.int32)
    o = wq.wq_decode_attention_fp8(qy.cuda(), kq.reshape(B, T, H, 128), ks, vq.reshape(B, T, H, 128), vs,
                                   lens.cuda())
    torch.cuda.synchronize()
    k_codes, k_s = kv.quantize_kv_fp8(kc.float().numpy())
    v_codes, v_s = kv.quantize_kv_fp8(vc.float().numpy())
    assert np.array_equal(kq.cpu().numpy().reshape(k_codes.shape), k_codes)
    assert np.array_equal(vq.cpu().numpy().reshape(v_codes.shape), v_codes)
    assert float(ks.item()) == float(k_s) and float(vs.item()) == float(v_s)
    o_ref, a_ref = kv.decode_attention(qy.float().numpy(), kv.dequant_kv_fp8(k_codes, k_s),
                                       kv.dequant_kv_fp8(v_codes, v_s), lengths)
    check_o(o, o_ref, a_ref)


@pytest.mark.parametrize("H,Hq", [(2, 16), (1, 1)])
def test_attention_fp8(H, Hq):
    fp8_case(3, 700, H, Hq, [700, 0, 129], 70 + H)


def test_attention_fp8_chunk_edges_and_70b_heads():
    fp8_case(4, 1100, 8, 64, [512, 513, 1, 1100], 80)
