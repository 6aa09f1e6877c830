"""SVDQuant W4A4 linear, written plainly in float64.

ORACLE -- test infrastructure only. Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the product package
never does.

What it computes (the Nunchaku README, "Method": the SVDQuant figure with its
three stages, and "Engine design": the 16-bit low-rank branch beside the 4-bit
compute, with down-projection sharing the quantizer's input and
up-projection sharing the 4-bit GEMM's output):

    Y = Q(X_hat) Q(R)^T + (X_hat L1) L2 + bias,   X_hat = X diag(smooth_inv)

Steps, each a function below:

a1  smooth        x_hat = RN32(x * smooth_inv[k])
a2  group scale   NVFP4: s = UE4M3(RN32(amax16 / 6));  INT4: s = FP16(RN32(amax64 / 7))
a3  quantize      NVFP4: q = E2M1(RN32(x_hat * RN32(1/s)))
                  INT4:  q = clamp(rint(RN32(x_hat * RN32(1/s))), -7, 7)
                  a group whose decoded scale is 0 stores scale 0 and codes 0
a4  down-proj     xl1 = x_hat @ L1 (x_hat as float32 values, exact sum in float64)
a5  4-bit GEMM    acc = dequant(codes_x) @ dequant(codes_w)^T
a6  up-proj       y = acc + xl1 @ L2 + bias

Group sizes: 16 along K for NVFP4 (Diffusers blog, "quantization_config":
``precision: nvfp4, group_size: 16``) and 64 for INT4 (the blog's int4
``group_size: 64``; symmetric with FP16 scales is the reading recorded in
the design notes).
"""

from __future__ import annotations

import numpy as np

from .formats import (e2m1_decode, e2m1_encode, fp16_round, rn32, ue4m3_decode,
                      ue4m3_encode, bf16_from_bits)

NVFP4 = "nvfp4"
INT4 = "int4"
GROUP = {NVFP4: 16, INT4: 64}


# ---------------------------------------------------------------- a1: smoothing
def smooth(x: np.ndarray, smooth_inv: np.ndarray | None) -> np.ndarray:
    """x_hat = RN32(x * smooth_inv) per input channel k (one float32 multiply).

    ``x`` holds bfloat16 values (exact in float64), ``smooth_inv`` float32
    values; ``None`` means no smoothing (x_hat = x, used for weights).
    """
    x = np.asarray(x, dtype=np.float64)
    if smooth_inv is None:
        return x.copy()
    return rn32(x * np.asarray(smooth_inv, dtype=np.float64)[None, :])


# ------------------------------------------------------- a2 + a3: quantization
def _groups(xhat: np.ndarray, g: int) -> np.ndarray:
    rows, K = xhat.shape
    if K % g:
        raise ValueError(f"K={K} is not a multiple of the group size {g}")
    return xhat.reshape(rows, K // g, g)


def quantize_nvfp4(xhat: np.ndarray):
    """NVFP4 group quantization of float32-valued ``xhat`` [rows, K].

    Returns (codes [rows, K] uint8 in 0..15, scale codes [rows, K/16] uint8 E4M3).
    """
    grp = _groups(xhat, 16)
    amax = np.max(np.abs(grp), axis=2)                     # exact
    s_code = ue4m3_encode(rn32(amax / 6.0))                # one f32 divide, then E4M3
    s_val = ue4m3_decode(s_code)
    zero = s_val == 0.0
    safe = np.where(zero, 1.0, s_val)
    rcp = rn32(1.0 / safe)                                 # correctly rounded f32 reciprocal
    q = e2m1_encode(rn32(grp * rcp[:, :, None]))           # one f32 multiply, then E2M1
    q = np.where(zero[:, :, None], np.uint8(0), q).astype(np.uint8)
    s_code = np.where(zero, np.uint8(0), s_code).astype(np.uint8)
    return q.reshape(xhat.shape), s_code


def quantize_int4(xhat: np.ndarray):
    """Symmetric INT4 group-64 quantization of float32-valued ``xhat`` [rows, K].

    Returns (codes [rows, K] int8 in -7..7, scales [rows, K/64] float64 holding FP16 values).
    """
    grp = _groups(xhat, 64)
    amax = np.max(np.abs(grp), axis=2)
    s = fp16_round(rn32(amax / 7.0))
    zero = s == 0.0
    safe = np.where(zero, 1.0, s)
    rcp = rn32(1.0 / safe)
    q = np.clip(np.rint(rn32(grp * rcp[:, :, None])), -7, 7)
    q = np.where(zero[:, :, None], 0.0, q)
    return q.reshape(xhat.shape).astype(np.int8), np.where(zero, 0.0, s)


# ------------------------------------------- two-level NVFP4 (per-tensor scale)
# The NVFP4 format named on the pages (Diffusers blog, "quantization_config":
# precision nvfp4, group_size 16) has a second scale level above the E4M3 group
# scales: one float32 factor per tensor, so that a tensor whose range lies outside
# what E4M3 group scales reach (amax/6 above 448 or below 2^-9) still quantizes
# with the format's relative precision. The pages state no formula for it; the
# reading (recorded in the design notes) is the usual one:
#
#   s_t  = RN32(amax / (6 * 448)) if that is a normal float32, else 1
#   inv  = RN32(1 / s_t)
#   x'   = RN32(x_hat * inv), then the one-level NVFP4 quantization of x'
#   Y    = RN32(s_t,a * s_t,w) * (4-bit product) + (x_hat L1) L2 + bias
#
# with amax the largest |x_hat| of the tensor (x_hat = the smoothed activation;
# the residual weight for weights). The low-rank branch keeps x_hat unscaled.

NVFP4_TENSOR_RANGE = 6.0 * 448.0
_F32_MIN_NORMAL = 2.0 ** -126


def tensor_scale(xhat: np.ndarray):
    """(s_t, inv) of a float32-valued tensor, both float32 values as float64."""
    amax = float(np.max(np.abs(np.asarray(xhat, np.float64)))) if np.size(xhat) else 0.0
    s = float(rn32(np.float64(amax) / NVFP4_TENSOR_RANGE))
    if not s >= _F32_MIN_NORMAL:
        s = 1.0
    return s, float(rn32(np.float64(1.0) / s))


def quantize_nvfp4_two_level(xhat: np.ndarray, inv: float):
    """Two-level NVFP4: the one-level quantization of RN32(x_hat * inv)."""
    return quantize_nvfp4(rn32(np.asarray(xhat, np.float64) * np.float64(inv)))


def dequant_nvfp4_two_level(codes, s_code, s_t: float) -> np.ndarray:
    return dequant_nvfp4(codes, s_code) * np.float64(s_t)


def w4a4_linear_two_level(a_deq: np.ndarray, w_deq: np.ndarray, s_ta: float, s_tw: float,
                          xl1: np.ndarray | None, L2: np.ndarray | None,
                          bias: np.ndarray | None) -> np.ndarray:
    """Y = RN32(s_ta * s_tw) * (a_deq @ w_deq^T) + xl1 @ L2 + bias, float64 (unrounded).

    a_deq / w_deq are the one-level dequantized codes of the scaled tensors."""
    alpha = float(rn32(np.float64(s_ta) * np.float64(s_tw)))
    y = alpha * (np.asarray(a_deq, np.float64) @ np.asarray(w_deq, np.float64).T)
    if xl1 is not None and L2 is not None and np.asarray(L2).shape[0] > 0:
        y += np.asarray(xl1, np.float64) @ np.asarray(L2, np.float64)
    if bias is not None:
        y += np.asarray(bias, np.float64)[None, :]
    return y


def quantize(fmt: str, xhat: np.ndarray):
    if fmt == NVFP4:
        return quantize_nvfp4(xhat)
    if fmt == INT4:
        return quantize_int4(xhat)
    raise ValueError(fmt)


def dequant_nvfp4(codes: np.ndarray, s_code: np.ndarray) -> np.ndarray:
    rows, K = codes.shape
    v = e2m1_decode(codes).reshape(rows, K // 16, 16)
    return (v * ue4m3_decode(s_code)[:, :, None]).reshape(rows, K)


def dequant_int4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    rows, K = codes.shape
    v = np.asarray(codes, dtype=np.float64).reshape(rows, K // 64, 64)
    return (v * np.asarray(scales, dtype=np.float64)[:, :, None]).reshape(rows, K)


def dequant(fmt: str, codes, scales) -> np.ndarray:
    return dequant_nvfp4(codes, scales) if fmt == NVFP4 else dequant_int4(codes, scales)


# ------------------------------------------------------------------- packing
def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte along K: element 2j in the low nibble, 2j+1 in the high.

    INT4 codes are stored as two's-complement nibbles.
    """
    c = (np.asarray(codes).astype(np.int16) & 0xF).astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray, signed: bool = False) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    if signed:
        s = out.astype(np.int8)
        return np.where(s >= 8, s - 16, s).astype(np.int8)
    return out


# ---------------------------------------------------------- a4 / a5 / a6: linear
def down_proj(xhat: np.ndarray, L1: np.ndarray) -> np.ndarray:
    """xl1 = x_hat @ L1 (float64; every product of an f32 and a bf16 is exact)."""
    return np.asarray(xhat, np.float64) @ np.asarray(L1, np.float64)


def w4a4_linear(a_deq: np.ndarray, w_deq: np.ndarray, xl1: np.ndarray | None,
                L2: np.ndarray | None, bias: np.ndarray | None) -> np.ndarray:
    """Y = a_deq @ w_deq^T + xl1 @ L2 + bias, all float64 (unrounded)."""
    y = np.asarray(a_deq, np.float64) @ np.asarray(w_deq, np.float64).T
    if xl1 is not None and L2 is not None and np.asarray(L2).shape[0] > 0:
        y += np.asarray(xl1, np.float64) @ np.asarray(L2, np.float64)
    if bias is not None:
        y += np.asarray(bias, np.float64)[None, :]
    return y


def w4a4_linear_rows(rows: np.ndarray, a_deq, w_deq, xl1, L2, bias) -> np.ndarray:
    """The same Y restricted to the given output rows (for sampled checks)."""
    rows = np.asarray(rows)
    return w4a4_linear(a_deq[rows], w_deq, None if xl1 is None else xl1[rows], L2, bias)


def svdq_forward(fmt: str, x_bits: np.ndarray, smooth_inv, L1, L2, w_codes, w_scales,
                 bias_bits=None) -> dict:
    """All of a1..a6 for activations given as bf16 bits; weights already quantized."""
    x = bf16_from_bits(x_bits)
    xhat = smooth(x, smooth_inv)
    codes, scales = quantize(fmt, xhat)
    xl1 = down_proj(xhat, L1) if L1 is not None and np.asarray(L1).shape[1] > 0 else None
    a_deq = dequant(fmt, codes, scales)
    w_deq = dequant(fmt, w_codes, w_scales)
    bias = None if bias_bits is None else bf16_from_bits(bias_bits)
    y = w4a4_linear(a_deq, w_deq, xl1, L2, bias)
    return {"xhat": xhat, "codes": codes, "scales": scales, "xl1": xl1, "Y": y}
