"""The fused MLP (fc1 -> GELU -> fc2) of an SVDQ transformer block, written
plainly in float64.

ORACLE -- test infrastructure only. Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the product package
never does.

What it computes (Diffusers blog, "From SVDQuant to Nunchaku Lite": the
original Nunchaku engine runs the MLP as one fused GELU/MLP path, where Lite
runs the two SVDQ linears separately): fc1's epilogue applies GELU to its
output and hands fc2 its 4-bit input directly, so the hidden activation
[M, 4 x hidden] never goes to HBM in 16 bits:

    y1      = the fc1 SVDQ layer's output [M, N1]            (with bias)
    h       = RN32(GELU(y1))                                 (float32 hidden value)
    h_hat   = RN32(h * smooth_inv2[n])                       (fc2's smoothing, step a1)
    codes, scales = NVFP4 quantization of h_hat              (steps a2, a3; groups along N1)
    xl1_2   = h_hat @ L1_2                                   (fc2's down-projection, step a4)
    y2      = the fc2 layer on (codes, scales, xl1_2)        (steps a5, a6)

The pages name the fused path but not its arithmetic; the readings this
follows: GELU is the tanh form 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3)))
that FLUX-style feed-forward blocks use (the erf form is kept beside it for the
pins); the hidden value is one float32 rounding of GELU of the exact fc1
output, with no bf16 rounding between fc1 and fc2 (the unfused pipeline
rounds fc1's output to bf16 before GELU and GELU's output to bf16 before fc2's
quantizer); fc2's smoothing and quantization are steps a1-a4 unchanged.
"""

from __future__ import annotations

import math

import numpy as np

from .formats import rn32
from .svdq import dequant_nvfp4, down_proj, quantize_nvfp4, w4a4_linear

_SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)


def gelu(y: np.ndarray, approximate: str = "tanh") -> np.ndarray:
    """GELU in float64: the tanh form, or the exact y Phi(y) with Phi via erf."""
    y = np.asarray(y, np.float64)
    if approximate == "tanh":
        return 0.5 * y * (1.0 + np.tanh(_SQRT_2_OVER_PI * (y + 0.044715 * y ** 3)))
    if approximate == "none":
        erf = np.vectorize(math.erf, otypes=[np.float64])
        return 0.5 * y * (1.0 + erf(y / math.sqrt(2.0)))
    raise ValueError(approximate)


def hidden(y1: np.ndarray, smooth_inv2: np.ndarray | None, approximate: str = "tanh") -> np.ndarray:
    """h_hat = RN32(RN32(GELU(y1)) * smooth_inv2), float32 values as float64."""
    h = rn32(gelu(y1, approximate))
    if smooth_inv2 is None:
        return h
    return rn32(h * np.asarray(smooth_inv2, np.float64)[None, :])


def fc1_epilogue(y1: np.ndarray, smooth_inv2, L1_2, approximate: str = "tanh") -> dict:
    """What fc1's fused epilogue emits for fc2: h_hat, its NVFP4 codes and scales, and xl1_2."""
    h_hat = hidden(y1, smooth_inv2, approximate)
    codes, scales = quantize_nvfp4(h_hat)
    xl1 = None
    if L1_2 is not None and np.asarray(L1_2).shape[1] > 0:
        xl1 = down_proj(h_hat, L1_2)
    return {"h_hat": h_hat, "codes": codes, "scales": scales, "xl1": xl1}


def mlp_forward(y1: np.ndarray, smooth_inv2, L1_2, L2_2, w2_codes, w2_scales, bias2,
                approximate: str = "tanh") -> dict:
    """fc2 of the fused MLP on fc1's output y1 (float64): fc1's epilogue, then steps a5, a6."""
    ep = fc1_epilogue(y1, smooth_inv2, L1_2, approximate)
    y2 = w4a4_linear(dequant_nvfp4(ep["codes"], ep["scales"]), dequant_nvfp4(w2_codes, w2_scales),
                     ep["xl1"], L2_2, bias2)
    return {**ep, "Y": y2}
