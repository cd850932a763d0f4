"""Offline activation-aware scale search (AWQ-style) driven through libwq's kernels.

"Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache Quantization", section "The methods
compared": AWQ finds the salient input channels from activation magnitudes and scales them up before
quantising; scaling can raise a group's maximum, so implementations search for the scale per channel.
"Test-time quantization: quantising on the fly with no calibration dataset", section "The idea": the
activations compensate for the rescaling (divided by the same scales), so the product is unchanged up to
the quantisation; AWQ takes the activation statistics offline, over a calibration set.

The scale of channel c is s_c = m_c ** alpha with m_c the mean |x[m][c]| over the calibration rows,
normalised so that max(s) * min(s) = 1; alpha runs over a grid and the value whose quantised product is
closest, in squared error over the calibration rows, to the exact product wins.  Every step on the data runs
in libwq's kernels: the channel magnitudes (wq_awq_channel_magnitudes, once) and, for each alpha, the scales
(wq_awq_channel_scales), the weights w[n][c] * s_c quantised (wq_quantize_int4_scaled) and the calibration
rows divided by s inside the matmul (wq_gemm_w4a16_colscaled).  The exact reference product and the squared
errors are the offline search's bookkeeping (binary64 on the host, one reference product per search).  At
decode time the same col_scale goes to wq_gemm_w4a16_colscaled, or the layer that produces x absorbs 1 / s,
as the pages say AWQ's scales are absorbed into neighbouring layers.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (wq_awq_channel_magnitudes, wq_awq_channel_scales, wq_gemm_w4a16_colscaled,
               wq_quantize_int4_scaled)

GRID = tuple(i / 20 for i in range(21))


def search(w: torch.Tensor, x_cal: torch.Tensor, g: int = 128, grid=GRID):
    """w: [N][K] float32 or bfloat16 on CUDA; x_cal: [M][K] bf16 calibration activations (any device).
    Returns (alpha, s float32 [K] numpy, errors list aligned with grid)."""
    if not w.is_cuda:
        raise TypeError("w must be a CUDA tensor (the statistics, quantiser and matmul run on the GPU)")
    x = x_cal.detach().to(torch.bfloat16).contiguous().to(w.device)
    mag = wq_awq_channel_magnitudes(x)
    exact = x.double().cpu().numpy() @ w.detach().double().cpu().numpy().T
    errors, scales = [], []
    for a in grid:
        s = wq_awq_channel_scales(mag, a)
        q, sc, z = wq_quantize_int4_scaled(w, s, g)
        y = wq_gemm_w4a16_colscaled(x, s, q, sc, z, g)
        errors.append(float(np.sum((y.double().cpu().numpy() - exact) ** 2)))
        scales.append(s)
    best = int(np.argmin(errors))
    return grid[best], scales[best].cpu().numpy(), errors
