"""The AWQ search's orchestration on the CPU: the library calls are replaced by the oracle's statistics,
quantiser and matmul (CPU tensors), so the loop, the scales and the bookkeeping run without a GPU.  The GPU
run of the same search is a parity test in test_gpu_parity.py."""
import numpy as np
import torch

import oracle
import wq_inputs
from oracle import awq as oawq


def _fake_magnitudes(x):
    return torch.from_numpy(oawq.channel_magnitude(x.double().numpy()))


def _fake_scales(mag, alpha):
    return torch.from_numpy(oawq.channel_scales(mag.numpy(), alpha))


def _fake_quantize_scaled(w, col_scale, g):
    codes, s, z = oracle.quantize_int4(oawq.scaled_weights(w.float().numpy(), col_scale.numpy()), g)
    return torch.from_numpy(codes), torch.from_numpy(s), torch.from_numpy(z)


def scaled_x(x, s):
    """bf16(x / s) with a binary32 quotient, as the library's kernels stage it."""
    q = (x.float().numpy() / s.astype(np.float32)[None, :]).astype(np.float32)
    return oracle.bf16_value(oracle.bf16_bits(q)).astype(np.float64)


def _fake_gemm_colscaled(x, col_scale, codes, s, z, g):
    y, _ = oracle.gemm_w4a16(scaled_x(x, col_scale.numpy()), codes.numpy(), s.numpy(), z.numpy(), g)
    return torch.from_numpy(y).to(torch.bfloat16)


def test_search_orchestration_matches_the_oracle_search(monkeypatch):
    import group_wise_weight_b200.awq as gawq
    monkeypatch.setattr(gawq, "wq_awq_channel_magnitudes", _fake_magnitudes)
    monkeypatch.setattr(gawq, "wq_awq_channel_scales", _fake_scales)
    monkeypatch.setattr(gawq, "wq_quantize_int4_scaled", _fake_quantize_scaled)
    monkeypatch.setattr(gawq, "wq_gemm_w4a16_colscaled", _fake_gemm_colscaled)

    class _CudaLike(torch.Tensor):  # the search insists on CUDA weights; the fakes take CPU tensors
        @property
        def is_cuda(self):
            return True

    w = wq_inputs.llm_weight(96, 512, 401, dtype=torch.float32)
    x = wq_inputs.activations(40, 512, 402, channel_seed=401)
    alpha, s, errors = gawq.search(w.as_subclass(_CudaLike), x, 128)
    assert len(errors) == len(gawq.GRID) and alpha == gawq.GRID[int(np.argmin(errors))]
    assert np.array_equal(s, oawq.channel_scales(oawq.channel_magnitude(x.double().numpy()), alpha))

    def deq(w32):
        codes, so, zo = oracle.quantize_int4(w32, 128)
        return oracle.dequant_int4(codes, so, zo, 128)
    o_alpha, _, o_errors = oawq.search(x.double().numpy(), w.numpy(), deq)
    # the orchestrated errors differ from the oracle's only by bf16 rounding of x / s and of y
    assert np.allclose(errors, o_errors, rtol=0.05)
    assert o_errors[gawq.GRID.index(alpha)] <= 1.05 * min(o_errors)
    assert alpha > 0
