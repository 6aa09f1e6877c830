"""AWQ W4A16 linear, plainly in float64.

ORACLE -- test infrastructure only.

The Diffusers blog, "From SVDQuant to Nunchaku Lite" and "quantization_config":
``awq_w4a16`` layers (modulation / adaptive-norm projections) keep 16-bit
activations and 4-bit weights, ``precision: int4, group_size: 64``.

Reading (asymmetric, the usual AWQ form): per group of 64 weights along K,
    s = BF16((max - min) / 15), s = 1 if max == min
    z = clamp(rint(-min / s), 0, 15)            (an integer, exact in bf16; zero is +0)
    q = clamp(rint(w / s + z), 0, 15)
and the layer computes y[m, n] = sum_k x[m, k] (q[n, k] - z[n, g]) s[n, g] + b[n].
The activation-aware scale search needs calibration data and is not part of it.
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_round

GROUP = 64


def quantize_weight(w: np.ndarray):
    """w [N, K] -> (q uint8 [N, K] in 0..15, s [N, K/64], z [N, K/64]) (bf16 values)."""
    w = np.asarray(w, np.float64)
    N, K = w.shape
    g = w.reshape(N, K // GROUP, GROUP)
    mx, mn = g.max(axis=2), g.min(axis=2)
    s = np.where(mx == mn, 1.0, bf16_round((mx - mn) / 15.0))
    z = np.clip(np.rint(-mn / s), 0, 15) + 0.0  # an integer: a zero point of zero is +0
    q = np.clip(np.rint(g / s[:, :, None] + z[:, :, None]), 0, 15)
    return q.reshape(N, K).astype(np.uint8), s, z


def dequant_weight(q, s, z) -> np.ndarray:
    q = np.asarray(q, np.float64)
    N, K = q.shape
    g = q.reshape(N, K // GROUP, GROUP)
    return ((g - np.asarray(z)[:, :, None]) * np.asarray(s)[:, :, None]).reshape(N, K)


def linear(x: np.ndarray, q, s, z, bias=None) -> np.ndarray:
    """y = x @ dequant(q, s, z)^T + bias, float64 (unrounded)."""
    y = np.asarray(x, np.float64) @ dequant_weight(q, s, z).T
    if bias is not None:
        y += np.asarray(bias, np.float64)[None, :]
    return y
