"""Offline weight preparation on the GPU (not part of the timed hot path).

Stages 2 and 3 of SVDQuant (Nunchaku README, "Method"): smooth the weights
with lambda, split W_hat by SVD into 16-bit factors L1 L2, and quantize the
residual R = W_hat - (L1 L2)^T with the library's own group quantizer. The
smoothing factor is lambda_k = sqrt(max |X_k| / max |W_k|) from calibration
activation maxima; the factor split is L1 = V_r sqrt(S_r), L2 = sqrt(S_r) U_r^T.

The library computes the smoothing vector (svdq_smoothing), the bf16 factors
from the SVD (svdq_lowrank_factors), the residual (svdq_residual, float64
inside) and its quantization, the low-rank operand and
the AWQ weight quantizer (awq_quantize_weight). The SVD of W_hat runs in torch
(cuSOLVER, float64), once per layer, offline, like the calibration tooling that
would produce a checkpoint.
"""

from __future__ import annotations

import torch

from . import (awq_quantize_weight, svdq_lowrank_factors, svdq_pack_lowrank, svdq_quantize_act,
               svdq_quantize_act_two_level, svdq_residual, svdq_smoothing, svdq_tensor_scale)


def smoothing(x_absmax: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    """smooth_inv [K] float32 = RN32(1 / lambda) (svdq_smoothing)."""
    return svdq_smoothing(x_absmax.float().contiguous(), w.contiguous())


def smoothed_weight(w: torch.Tensor, x_absmax: torch.Tensor):
    """(smooth_inv [K] f32, W_hat = W diag(1 / smooth_inv) [N, K] float64), the SVD's input."""
    smooth_inv = smoothing(x_absmax, w)
    return smooth_inv, w.double() * (1.0 / smooth_inv.double())[None, :]


def prepare_svdq_weights(w: torch.Tensor, x_absmax: torch.Tensor, rank: int,
                         fmt: str = "nvfp4", two_level: bool = False, svd=None) -> dict:
    """w [N, K] bf16 (nn.Linear layout), x_absmax [K] per-channel max |X|.

    Returns device tensors: smooth_inv [K] f32, L1 [K, r] bf16, L1s [2, r, K] bf16
    (the down-projection operand), L2 [r, N] bf16, w_codes, w_scales (tiled), and
    R [N, K] bf16 (the quantized residual's input). With ``two_level`` (NVFP4 only)
    the residual is quantized with its own per-tensor scale, returned as w_tscale
    (float32 [2]: s_t, 1 / s_t); otherwise w_tscale is None. ``svd`` may pass
    (U, S, V^T) of smoothed_weight's W_hat, to share one decomposition between
    the ranks of one weight; by default it is computed here in float64.
    """
    if two_level and fmt != "nvfp4":
        raise ValueError("two-level scaling is an NVFP4 format")
    N, K = w.shape
    smooth_inv, w_hat = smoothed_weight(w, x_absmax)
    if rank > 0:
        u, s, vh = svd if svd is not None else torch.linalg.svd(w_hat, full_matrices=False)
        L1, L2 = svdq_lowrank_factors(u.double(), s.double(), vh.double(), rank)  # [K, r], [r, N]
        L1s = svdq_pack_lowrank(L1, smooth_inv.contiguous())
    else:
        L1 = L1s = L2 = None
    R = svdq_residual(w.contiguous(), smooth_inv, L1, L2)
    if two_level:
        w_tscale = svdq_tensor_scale(R)
        w_codes, w_scales, _ = svdq_quantize_act_two_level(R, w_tscale)
    else:
        w_tscale = None
        w_codes, w_scales, _ = svdq_quantize_act(R, None, None, fmt=fmt)
    return {"smooth_inv": smooth_inv.contiguous(), "L1": L1, "L1s": L1s,
            "L2": L2.contiguous() if L2 is not None else None, "w_codes": w_codes, "w_scales": w_scales,
            "w_tscale": w_tscale, "R": R, "fmt": fmt, "N": N, "K": K, "r": rank}


def prepare_awq_weights(w: torch.Tensor) -> dict:
    """w [N, K] bf16 -> fragment-ordered qweight and interleaved (scale, zero) (awq_quantize_weight)."""
    N, K = w.shape
    qt, szt = awq_quantize_weight(w.contiguous())
    return {"qweight": qt, "sz": szt, "N": N, "K": K}
