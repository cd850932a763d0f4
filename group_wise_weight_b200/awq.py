"""Offline activation-aware scale search (AWQ-style) driven through libwq's kernels.

"Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache Quantization", section "The methods
compared": AWQ finds the salient input channels from activation magnitudes and scales them up before
quantising; scaling can raise a group's maximum, so implementations search for the scale per channel.
"Test-time quantization: quantising on the fly with no calibration dataset", section "The idea": the
activations compensate for the rescaling (divided by the same scales), so the product is unchanged up to
the quantisation; AWQ takes the activation statistics offline, over a calibration set.

The scale of channel c is s_c = m_c ** alpha with m_c the mean |x[m][c]| over the calibration rows,
normalised so that max(s) * min(s) = 1; alpha runs over a grid and the value whose quantised product is
closest, in squared error over the calibration rows, to the exact product wins.  For each alpha the
weights are quantised by wq_quantize_int4_scaled (w[n][c] * s_c in binary32 on the GPU) and the
calibration rows, divided by s and rounded to bf16, go through wq_gemm_w4a16.  The statistics, the exact
reference product and the squared errors are host-side bookkeeping of this offline search (binary64); the
decode-time path is unchanged: the layer that produces x is expected to absorb 1 / s, as the pages say
AWQ's scales are absorbed into neighbouring layers.
"""
from __future__ import annotations

import numpy as np
import torch

from . import wq_gemm_w4a16, wq_quantize_int4_scaled

GRID = tuple(i / 20 for i in range(21))


def channel_scales(magnitude: np.ndarray, alpha: float) -> np.ndarray:
    """s_c = m_c ** alpha, normalised to max * min = 1; a silent channel (m_c = 0) takes the smallest
    positive magnitude.  float32, the precision the weights are scaled in."""
    m = np.asarray(magnitude, dtype=np.float64)
    pos = m[m > 0]
    s = np.where(m > 0, m, pos.min() if pos.size else 1.0) ** alpha
    return (s / np.sqrt(s.max() * s.min())).astype(np.float32)


def search(w: torch.Tensor, x_cal: torch.Tensor, g: int = 128, grid=GRID):
    """w: [N][K] float32 or bfloat16 on CUDA; x_cal: [M][K] calibration activations (any device).
    Returns (alpha, s float32 [K] numpy, errors list aligned with grid)."""
    if not w.is_cuda:
        raise TypeError("w must be a CUDA tensor (the quantiser and the matmul run on the GPU)")
    x64 = x_cal.detach().double().cpu().numpy()
    mag = np.mean(np.abs(x64), axis=0)
    exact = x64 @ w.detach().double().cpu().numpy().T
    errors = []
    for a in grid:
        s = channel_scales(mag, a)
        q, sc, z = wq_quantize_int4_scaled(w, torch.from_numpy(s).to(w.device), g)
        xs = torch.from_numpy((x64 / s.astype(np.float64)).astype(np.float32)).to(torch.bfloat16).to(w.device)
        y = wq_gemm_w4a16(xs, q, sc, z, g)
        errors.append(float(np.sum((y.double().cpu().numpy() - exact) ** 2)))
    best = int(np.argmin(errors))
    return grid[best], channel_scales(mag, grid[best]), errors
