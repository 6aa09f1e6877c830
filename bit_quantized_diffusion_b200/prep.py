"""Offline weight preparation on the GPU (not part of the timed hot path).

Stages 2 and 3 of SVDQuant (Nunchaku README, "Method"): smooth the weights
with lambda, split W_hat by SVD into 16-bit factors L1 L2, and quantize the
residual R = W_hat - (L1 L2)^T with the library's own group quantizer. The
smoothing factor is lambda_k = sqrt(max |X_k| / max |W_k|) from calibration
activation maxima; the factor split is L1 = V_r sqrt(S_r), L2 = sqrt(S_r) U_r^T.

The SVD and the dense residual use torch linear algebra (cuSOLVER / cuBLAS):
this runs once per layer, offline, like the calibration tooling that would
produce a checkpoint. The quantization of R and all packing run in libsvdq.

Also the AWQ W4A16 weight quantizer (asymmetric int4, group 64, bf16 scale and
zero) followed by the fragment-order pack.
"""

from __future__ import annotations

import torch

from . import (svdq_pack, svdq_pack_lowrank, svdq_quantize_act, svdq_quantize_act_two_level,
               svdq_tensor_scale)


def smoothing(x_absmax: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    """smooth_inv [K] float32 = 1 / lambda."""
    wmax = w.float().abs().amax(dim=0)
    xmax = x_absmax.float()
    ok = (xmax > 0) & (wmax > 0)
    lam = torch.where(ok, torch.sqrt(torch.where(ok, xmax, 1.0) / torch.where(ok, wmax, 1.0)),
                      torch.ones_like(xmax))
    return (1.0 / lam.double()).float()


def prepare_svdq_weights(w: torch.Tensor, x_absmax: torch.Tensor, rank: int,
                         fmt: str = "nvfp4", two_level: bool = False) -> dict:
    """w [N, K] bf16 (nn.Linear layout), x_absmax [K] per-channel max |X|.

    Returns device tensors: smooth_inv [K] f32, L1 [K, r] bf16, L1s [2, r, K] bf16
    (the down-projection operand), L2 [r, N] bf16, w_codes, w_scales (tiled), and
    R [N, K] bf16 (the quantized residual's input). With ``two_level`` (NVFP4 only)
    the residual is quantized with its own per-tensor scale, returned as w_tscale
    (float32 [2]: s_t, 1 / s_t); otherwise w_tscale is None.
    """
    if two_level and fmt != "nvfp4":
        raise ValueError("two-level scaling is an NVFP4 format")
    N, K = w.shape
    smooth_inv = smoothing(x_absmax, w)
    w_hat = w.double() / smooth_inv.double()[None, :]
    if rank > 0:
        u, s, vh = torch.linalg.svd(w_hat, full_matrices=False)
        root = torch.sqrt(s[:rank])
        L1 = (vh[:rank].T * root[None, :]).to(torch.bfloat16)          # [K, r]
        L2 = (root[:, None] * u[:, :rank].T).to(torch.bfloat16)         # [r, N]
        R = (w_hat - (L1.double() @ L2.double()).T).to(torch.bfloat16)
        L1 = L1.contiguous()
        L1s = svdq_pack_lowrank(L1, smooth_inv.contiguous())
    else:
        L1 = L1s = L2 = None
        R = w_hat.to(torch.bfloat16)
    R = R.contiguous()
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
    """w [N, K] bf16 -> fragment-ordered qweight and interleaved (scale, zero)."""
    N, K = w.shape
    g = w.double().reshape(N, K // 64, 64)
    mx, mn = g.amax(dim=2), g.amin(dim=2)
    s = torch.where(mx == mn, torch.ones_like(mx), ((mx - mn) / 15.0).to(torch.bfloat16).double())
    z = torch.clamp(torch.round(-mn / s), 0, 15)
    q = torch.clamp(torch.round(g / s[:, :, None] + z[:, :, None]), 0, 15).to(torch.uint8)
    q = q.reshape(N, K)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).contiguous().reshape(-1)
    s16 = s.to(torch.bfloat16).contiguous()
    z16 = z.to(torch.bfloat16).contiguous()
    qt, szt = svdq_pack("awq", "nvfp4", N, K, packed, s16.view(torch.uint8).reshape(-1),
                        z16.view(torch.uint8).reshape(-1))
    return {"qweight": qt, "sz": szt, "N": N, "K": K}
