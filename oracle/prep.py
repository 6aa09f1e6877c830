"""Offline weight preparation (stages 2 and 3 of SVDQuant), plainly in float64.

ORACLE -- test infrastructure only.

The Nunchaku README, "Method" (the SVDQuant figure): stage 2 migrates
activation outliers into the weights, X_hat = X diag(lambda)^-1 and
W_hat = W diag(lambda); stage 3 splits W_hat by SVD into a low-rank part
L1 L2 kept in 16 bits and a residual R = W_hat - (L1 L2)^T that is quantized
to 4 bits.

Readings (the pages print no formulas for these):
* lambda_k = sqrt(max_m |X_mk| / max_n |W_nk|) (smoothing strength 0.5), and
  lambda_k = 1 when either maximum is 0. The kernels take
  smooth_inv = RN32(1 / lambda); W_hat uses lambda' = 1 / smooth_inv so that
  X_hat W_hat^T = X W^T up to the float32 rounding of x_hat.
* With W_hat = U S V^T: L1 = V_r sqrt(S_r) [K, r] and L2 = sqrt(S_r) U_r^T [r, N],
  each rounded once to bfloat16. R is formed from the rounded factors and
  rounded once to bfloat16 before it goes through the same group quantizer
  as the activations (no smoothing, rank 0).
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_from_bits, bf16_round, rn32
from .svdq import quantize


def smoothing_factors(x: np.ndarray, w: np.ndarray):
    """(lambda [K] float64, smooth_inv [K] float32 values as float64)."""
    xmax = np.max(np.abs(np.asarray(x, np.float64)), axis=0)
    wmax = np.max(np.abs(np.asarray(w, np.float64)), axis=0)
    ok = (xmax > 0) & (wmax > 0)
    lam = np.where(ok, np.sqrt(np.where(ok, xmax, 1.0) / np.where(ok, wmax, 1.0)), 1.0)
    return lam, rn32(1.0 / lam)


def svd_split(w_hat: np.ndarray, r: int):
    """Rank-r factors (L1 [K, r], L2 [r, N]) of W_hat [N, K], rounded to bfloat16."""
    N, K = w_hat.shape
    if r == 0:
        return np.zeros((K, 0)), np.zeros((0, N))
    u, s, vt = np.linalg.svd(np.asarray(w_hat, np.float64), full_matrices=False)
    root = np.sqrt(s[:r])
    L1 = bf16_round(vt[:r].T * root[None, :])
    L2 = bf16_round(root[:, None] * u[:, :r].T)
    return L1, L2


def residual(w_hat: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """R = W_hat - (L1 L2)^T, rounded once to bfloat16."""
    return bf16_round(w_hat - (L1 @ L2).T)


def prepare_svdq_layer(fmt: str, x_bits: np.ndarray, w_bits: np.ndarray, r: int) -> dict:
    """Everything the runtime layer needs, from bf16 X (calibration) and W."""
    x = bf16_from_bits(x_bits)
    w = bf16_from_bits(w_bits)
    lam, smooth_inv = smoothing_factors(x, w)
    w_hat = w * (1.0 / smooth_inv)[None, :]
    L1, L2 = svd_split(w_hat, r)
    R = residual(w_hat, L1, L2)
    w_codes, w_scales = quantize(fmt, R)
    return {"lambda": lam, "smooth_inv": smooth_inv, "w_hat": w_hat, "L1": L1, "L2": L2,
            "R": R, "w_codes": w_codes, "w_scales": w_scales}
