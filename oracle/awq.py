"""Activation-aware per-input-channel scaling before quantisation, AWQ-style (test infrastructure).

Only the test suite may import this; the CUDA library never does, and this module imports nothing of it.

What the pages fix, cited by page title and section:
  * "Quantization Methods Compared: INT8, GPTQ, AWQ, FP8, FP4 and KV-Cache Quantization" -- "The methods
    compared": AWQ finds the salient channels from activation magnitudes and scales them up before
    quantising, which gives them a finer effective resolution; scaling a channel up can raise its group's
    maximum, so real implementations search for the scale per channel.
  * "Test-time quantization: quantising on the fly with no calibration dataset" -- "The idea" (step 4):
    the activations compensate for the rescaling, so the product is unchanged; AWQ measures activation
    magnitudes over a calibration set in an offline pass.

Reading (the pages give no formula for the scale): one scale per input channel c,
    s_c = m_c ** alpha,  m_c = mean over the calibration rows of |x[m][c]|,
normalised so that max(s) * min(s) = 1, with alpha taken from the grid 0, 1/20, ..., 1 as the value
whose quantised product is closest, in squared error over the calibration rows, to the exact product.
The weights the quantiser sees are w[n][c] * s_c rounded to binary32; the activations that meet them
are x[m][c] / s_c.  alpha = 0 is plain quantisation.  Everything except the quantiser (the oracle's own,
binary32 as everywhere) runs in binary64.
"""
from __future__ import annotations

import numpy as np

GRID = tuple(i / 20 for i in range(21))


def channel_magnitude(x_cal) -> np.ndarray:
    """m_c = mean over rows of |x[m][c]|, binary64."""
    return np.mean(np.abs(np.asarray(x_cal, dtype=np.float64)), axis=0)


def channel_scales(magnitude, alpha: float) -> np.ndarray:
    """s_c = m_c ** alpha, normalised to max * min = 1; channels with m_c = 0 take the smallest positive
    magnitude (a scale of 0 cannot be compensated).  binary32, the precision the weights are scaled in."""
    m = np.asarray(magnitude, dtype=np.float64)
    pos = m[m > 0]
    floor = pos.min() if pos.size else 1.0
    s = np.where(m > 0, m, floor) ** alpha
    s = s / np.sqrt(s.max() * s.min())
    return s.astype(np.float32)


def scaled_weights(w, s) -> np.ndarray:
    """The weights the quantiser sees: w[n][c] * s_c, each product rounded to binary32."""
    return (np.asarray(w, dtype=np.float32) * np.asarray(s, dtype=np.float32)[None, :]).astype(np.float32)


def quantised_product(x, w_hat_scaled, s) -> np.ndarray:
    """y[m][n] = sum_c (x[m][c] / s_c) * w_hat'[n][c] in binary64 (the compensated product)."""
    xs = np.asarray(x, dtype=np.float64) / np.asarray(s, dtype=np.float64)[None, :]
    return xs @ np.asarray(w_hat_scaled, dtype=np.float64).T


def output_error(x, w, s, dequantised) -> float:
    """Squared error, over the rows of x, between the exact product x w^T and the quantised product of the
    scaled weights; `dequantised(w32)` returns the binary64 weights the quantiser reconstructs."""
    exact = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T
    got = quantised_product(x, dequantised(scaled_weights(w, s)), s)
    return float(np.sum((got - exact) ** 2))


def search(x_cal, w, dequantised, grid=GRID):
    """The grid search: returns (alpha, s, errors) with errors[i] the calibration error at grid[i]; the
    first minimum wins ties."""
    mag = channel_magnitude(x_cal)
    errors = [output_error(x_cal, w, channel_scales(mag, a), dequantised) for a in grid]
    best = int(np.argmin(errors))
    return grid[best], channel_scales(mag, grid[best]), errors
