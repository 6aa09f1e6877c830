"""B200 (sm_100a) SVDQuant W4A4 linear and AWQ W4A16 linear.

The compute lives in ``libsvdq.so`` (C ABI, include/svdq.h). This module is
the Python binding: one function per C call, with the same name, taking torch
CUDA tensors and marshalling pointers, sizes and the current stream. torch is
used for device memory and streams only.
"""

from __future__ import annotations

import torch

from . import _native as N
from ._native import SvdqError  # noqa: F401

FORMATS = {"nvfp4": N.NVFP4_G16, "int4": N.INT4_G64}
PACK_KINDS = {"act": N.PACK_ACT, "weight": N.PACK_WEIGHT, "awq": N.PACK_AWQ}


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def _ptr(t: torch.Tensor | None) -> int | None:
    """A tensor's device address. The library launches on the current device
    (and its tensor maps and static arrays are that device's), so a tensor on
    another device is refused here rather than read across devices."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"tensor on {t.device}, but the current device is cuda:{cur}: "
                         f"call under torch.cuda.device({t.device})")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, nbytes: int, name: str) -> None:
    if t.numel() * t.element_size() < nbytes:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, needs {nbytes}")


def svdq_codes_bytes(fmt, rows: int, K: int) -> int:
    return N.load().svdq_codes_bytes(_fmt(fmt), rows, K)


def svdq_scales_bytes(fmt, rows: int, K: int) -> int:
    return N.load().svdq_scales_bytes(_fmt(fmt), rows, K)


def awq_qweight_bytes(Nrows: int, K: int) -> int:
    return N.load().awq_qweight_bytes(Nrows, K)


def awq_sz_bytes(Nrows: int, K: int) -> int:
    return N.load().awq_sz_bytes(Nrows, K)


def svdq_xl1_splits(M: int, K: int, r: int) -> int:
    """S: svdq_quantize_act's xl1 buffer holds S x M x r float32 (its working space)."""
    return N.load().svdq_xl1_splits(M, K, r)


def svdq_quantize_act(X: torch.Tensor, L1s: torch.Tensor | None = None,
                      smooth_inv: torch.Tensor | None = None, fmt="nvfp4",
                      codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                      xl1: torch.Tensor | None = None, stream=None):
    """Steps a1..a4 on X [M, K] bf16. L1s is the [2, r, K] bf16 operand from
    svdq_pack_lowrank. xl1, if given, is a float32 buffer of at least
    svdq_xl1_splits(M, K, r) * M * r elements (the call's working space).
    Returns (codes, scales, xl1 [M, r] or None), xl1 a view of the buffer's start."""
    lib = N.load()
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise ValueError("X must be a 2-D bf16 tensor")
    M, K = X.shape
    r = 0 if L1s is None else L1s.shape[1]
    f = _fmt(fmt)
    dev = X.device
    if codes is None:
        codes = torch.empty(lib.svdq_codes_bytes(f, M, K), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(lib.svdq_scales_bytes(f, M, K), dtype=torch.uint8, device=dev)
    S = lib.svdq_xl1_splits(M, K, r) if r else 0
    if r and xl1 is None:
        xl1 = torch.empty((S, M, r), dtype=torch.float32, device=dev)
    _need(codes, lib.svdq_codes_bytes(f, M, K), "codes")
    _need(scales, lib.svdq_scales_bytes(f, M, K), "scales")
    if L1s is not None and (L1s.dtype != torch.bfloat16 or tuple(L1s.shape) != (2, r, K)):
        raise ValueError("L1s must be bf16 [2, r, K]")
    if smooth_inv is not None and (smooth_inv.dtype != torch.float32 or smooth_inv.numel() != K):
        raise ValueError("smooth_inv must be float32 [K]")
    if xl1 is not None and (xl1.dtype != torch.float32 or xl1.numel() < S * M * r):
        raise ValueError(f"xl1 must be float32 [{S}, M, r]")
    N.check(lib.svdq_quantize_act(f, M, K, r, _ptr(X), K, _ptr(smooth_inv), _ptr(L1s),
                                  _ptr(codes), _ptr(scales), _ptr(xl1) if r else None,
                                  _stream(stream)), "svdq_quantize_act")
    return codes, scales, (xl1.view(-1)[:M * r].view(M, r) if r else None)


def svdq_quantize_act_noalloc(X: torch.Tensor, L1s: torch.Tensor | None = None,
                              smooth_inv: torch.Tensor | None = None, fmt="nvfp4",
                              codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                              xl1: torch.Tensor | None = None, stream=None):
    """svdq_quantize_act with xl1 only [M, r] and no working space from the caller,
    for callers whose allocator cannot grant memory mid-step (a runtime or plugin
    that sized all device memory up front): the K splits' partial sums go to one
    static device array the library holds per device, (S - 1) * M * r <= 2^21
    floats; larger requests raise SvdqError. Two such calls that overlap on the
    GPU race on that array."""
    lib = N.load()
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise ValueError("X must be a 2-D bf16 tensor")
    M, K = X.shape
    r = 0 if L1s is None else L1s.shape[1]
    f = _fmt(fmt)
    dev = X.device
    if codes is None:
        codes = torch.empty(lib.svdq_codes_bytes(f, M, K), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(lib.svdq_scales_bytes(f, M, K), dtype=torch.uint8, device=dev)
    if r and xl1 is None:
        xl1 = torch.empty((M, r), dtype=torch.float32, device=dev)
    _need(codes, lib.svdq_codes_bytes(f, M, K), "codes")
    _need(scales, lib.svdq_scales_bytes(f, M, K), "scales")
    if L1s is not None and (L1s.dtype != torch.bfloat16 or tuple(L1s.shape) != (2, r, K)):
        raise ValueError("L1s must be bf16 [2, r, K]")
    if smooth_inv is not None and (smooth_inv.dtype != torch.float32 or smooth_inv.numel() != K):
        raise ValueError("smooth_inv must be float32 [K]")
    if xl1 is not None and (xl1.dtype != torch.float32 or xl1.numel() < M * r):
        raise ValueError("xl1 must be float32 [M, r]")
    N.check(lib.svdq_quantize_act_noalloc(f, M, K, r, _ptr(X), K, _ptr(smooth_inv), _ptr(L1s),
                                          _ptr(codes), _ptr(scales), _ptr(xl1) if r else None,
                                          _stream(stream)), "svdq_quantize_act_noalloc")
    return codes, scales, (xl1.view(-1)[:M * r].view(M, r) if r else None)


def svdq_pack_lowrank(L1: torch.Tensor, smooth_inv: torch.Tensor | None = None,
                      L1s: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """L1 [K, r] bf16 (+ smooth_inv [K] f32) -> the [2, r, K] bf16 down-projection operand."""
    lib = N.load()
    if L1.dtype != torch.bfloat16 or L1.dim() != 2:
        raise ValueError("L1 must be a 2-D bf16 tensor [K, r]")
    K, r = L1.shape
    if L1s is None:
        L1s = torch.empty((2, r, K), dtype=torch.bfloat16, device=L1.device)
    if smooth_inv is not None and (smooth_inv.dtype != torch.float32 or smooth_inv.numel() != K):
        raise ValueError("smooth_inv must be float32 [K]")
    N.check(lib.svdq_pack_lowrank(K, r, _ptr(L1), _ptr(smooth_inv), _ptr(L1s), _stream(stream)),
            "svdq_pack_lowrank")
    return L1s


def svdq_w4a4_linear(a_codes, a_scales, xl1, w_codes, w_scales, L2, bias, M: int, N_: int,
                     K: int, fmt="nvfp4", out_dtype=torch.bfloat16, Y: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Steps a5..a6: Y [M, N] = Q(X_hat) Q(R)^T + xl1 @ L2 + bias."""
    lib = N.load()
    r = 0 if L2 is None else L2.shape[0]
    if r and (xl1 is None or xl1.dtype != torch.float32 or xl1.numel() < M * r):
        raise ValueError("xl1 must be float32 [M, r]")
    f = _fmt(fmt)
    out = N.OUT_F32 if out_dtype == torch.float32 else N.OUT_BF16
    if Y is None:
        Y = torch.empty((M, N_), dtype=out_dtype, device=a_codes.device)
    if Y.dtype != out_dtype or Y.dim() != 2 or Y.shape[0] != M or Y.shape[1] < N_:
        raise ValueError("Y must be [M, >= N] of out_dtype")
    if L2 is not None and (L2.dtype != torch.bfloat16 or tuple(L2.shape) != (r, N_)):
        raise ValueError("L2 must be bf16 [r, N]")
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != N_):
        raise ValueError("bias must be bf16 [N]")
    _need(a_codes, lib.svdq_codes_bytes(f, M, K), "a_codes")
    _need(a_scales, lib.svdq_scales_bytes(f, M, K), "a_scales")
    _need(w_codes, lib.svdq_codes_bytes(f, N_, K), "w_codes")
    _need(w_scales, lib.svdq_scales_bytes(f, N_, K), "w_scales")
    N.check(lib.svdq_w4a4_linear(f, M, N_, K, r, _ptr(a_codes), _ptr(a_scales),
                                 _ptr(xl1) if r else None, _ptr(w_codes), _ptr(w_scales),
                                 _ptr(L2) if r else None, _ptr(bias), _ptr(Y), Y.shape[1], out,
                                 _stream(stream)), "svdq_w4a4_linear")
    return Y


def svdq_mlp_splits(M: int, N1: int) -> int:
    """S: svdq_mlp_fc1's xl1_2 buffer holds S x M x r2 float32 (its working space)."""
    return N.load().svdq_mlp_splits(M, N1)


def svdq_mlp_fc1(a_codes, a_scales, xl1_1, w_codes, w_scales, L2_1, bias1, smooth_inv2, L1t_2,
                 M: int, N1: int, K1: int, codes2=None, scales2=None, xl1_2=None, hhat=None, stream=None):
    """The fused MLP's fc1 (NVFP4): fc1's layer, GELU (tanh form), fc2's smoothing and
    fc2's activation quantization and down-projection in the epilogue. L1t_2 is fc2's
    factor transposed, bf16 [r2, N1] (or None for r2 = 0). hhat, if given, receives
    h_hat float32 [M, N1]. Returns (codes2, scales2, xl1_2 [M, r2] or None): fc2's input."""
    lib = N.load()
    r1 = 0 if L2_1 is None else L2_1.shape[0]
    r2 = 0 if L1t_2 is None else L1t_2.shape[0]
    dev = a_codes.device
    if r1 and (xl1_1 is None or xl1_1.dtype != torch.float32 or xl1_1.numel() < M * r1):
        raise ValueError("xl1_1 must be float32 [M, r1]")
    if r1 and (L2_1.dtype != torch.bfloat16 or tuple(L2_1.shape) != (r1, N1)):
        raise ValueError("L2_1 must be bf16 [r1, N1]")
    if r2 and (L1t_2.dtype != torch.bfloat16 or tuple(L1t_2.shape) != (r2, N1)):
        raise ValueError("L1t_2 must be bf16 [r2, N1]")
    if smooth_inv2 is not None and (smooth_inv2.dtype != torch.float32 or smooth_inv2.numel() != N1):
        raise ValueError("smooth_inv2 must be float32 [N1]")
    if bias1 is not None and (bias1.dtype != torch.bfloat16 or bias1.numel() != N1):
        raise ValueError("bias1 must be bf16 [N1]")
    S = lib.svdq_mlp_splits(M, N1)
    if S < 1:
        raise ValueError("N1 must be a positive multiple of 128")
    if codes2 is None:
        codes2 = torch.empty(lib.svdq_codes_bytes(N.NVFP4_G16, M, N1), dtype=torch.uint8, device=dev)
    if scales2 is None:
        scales2 = torch.empty(lib.svdq_scales_bytes(N.NVFP4_G16, M, N1), dtype=torch.uint8, device=dev)
    _need(codes2, lib.svdq_codes_bytes(N.NVFP4_G16, M, N1), "codes2")
    _need(scales2, lib.svdq_scales_bytes(N.NVFP4_G16, M, N1), "scales2")
    if r2 and xl1_2 is None:
        xl1_2 = torch.empty((S, M, r2), dtype=torch.float32, device=dev)
    if r2 and (xl1_2.dtype != torch.float32 or xl1_2.numel() < S * M * r2):
        raise ValueError(f"xl1_2 must be float32 [{S}, M, r2]")
    if hhat is not None and (hhat.dtype != torch.float32 or hhat.numel() < M * N1):
        raise ValueError("hhat must be float32 [M, N1]")
    N.check(lib.svdq_mlp_fc1(M, N1, K1, r1, r2, _ptr(a_codes), _ptr(a_scales), _ptr(xl1_1) if r1 else None,
                             _ptr(w_codes), _ptr(w_scales), _ptr(L2_1), _ptr(bias1), _ptr(smooth_inv2),
                             _ptr(L1t_2), _ptr(codes2), _ptr(scales2), _ptr(xl1_2) if r2 else None,
                             _ptr(hhat), _stream(stream)), "svdq_mlp_fc1")
    return codes2, scales2, (xl1_2.view(-1)[:M * r2].view(M, r2) if r2 else None)


def svdq_w4a4_linear_qkv_norm_rope(a_codes, a_scales, xl1, w_codes, w_scales, L2, bias, norm_q,
                                   norm_k, rope_cos, rope_sin, M: int, N_: int, K: int,
                                   eps: float = 1e-6, out_dtype=torch.bfloat16,
                                   Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The fused QKV projection (NVFP4): Y [M, N] = Q(X_hat) Q(R)^T + xl1 @ L2 + bias with
    every 128-column head of Q and K (columns [0, N/3) and [N/3, 2N/3)) RMS-normalised
    (norm_q / norm_k bf16 [128] or None, eps) and then turned pairwise by rope_cos /
    rope_sin float32 [64, M], angle-major (angle i of row m at [i, m]; both None: no
    rotation); V unchanged. N % 384 == 0."""
    lib = N.load()
    r = 0 if L2 is None else L2.shape[0]
    if r and (xl1 is None or xl1.dtype != torch.float32 or xl1.numel() < M * r):
        raise ValueError("xl1 must be float32 [M, r]")
    out = N.OUT_F32 if out_dtype == torch.float32 else N.OUT_BF16
    if Y is None:
        Y = torch.empty((M, N_), dtype=out_dtype, device=a_codes.device)
    if Y.dtype != out_dtype or Y.dim() != 2 or Y.shape[0] != M or Y.shape[1] < N_:
        raise ValueError("Y must be [M, >= N] of out_dtype")
    if L2 is not None and (L2.dtype != torch.bfloat16 or tuple(L2.shape) != (r, N_)):
        raise ValueError("L2 must be bf16 [r, N]")
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != N_):
        raise ValueError("bias must be bf16 [N]")
    for g, name in ((norm_q, "norm_q"), (norm_k, "norm_k")):
        if g is not None and (g.dtype != torch.bfloat16 or g.numel() != 128 or not g.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 [128]")
    for tb, name in ((rope_cos, "rope_cos"), (rope_sin, "rope_sin")):
        if tb is not None and (tb.dtype != torch.float32 or tuple(tb.shape) != (64, M)
                               or not tb.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous float32 [64, M] (angle-major)")
    f = N.NVFP4_G16
    _need(a_codes, lib.svdq_codes_bytes(f, M, K), "a_codes")
    _need(a_scales, lib.svdq_scales_bytes(f, M, K), "a_scales")
    _need(w_codes, lib.svdq_codes_bytes(f, N_, K), "w_codes")
    _need(w_scales, lib.svdq_scales_bytes(f, N_, K), "w_scales")
    N.check(lib.svdq_w4a4_linear_qkv_norm_rope(
        M, N_, K, r, _ptr(a_codes), _ptr(a_scales), _ptr(xl1) if r else None, _ptr(w_codes),
        _ptr(w_scales), _ptr(L2) if r else None, _ptr(bias), _ptr(norm_q), _ptr(norm_k),
        float(eps), _ptr(rope_cos), _ptr(rope_sin), _ptr(Y), Y.shape[1], out, _stream(stream)),
        "svdq_w4a4_linear_qkv_norm_rope")
    return Y


def svdq_tensor_scale(X: torch.Tensor, smooth_inv: torch.Tensor | None = None,
                      scale: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Two-level NVFP4: float32 [2] = (s_t, RN32(1 / s_t)) of x_hat = RN32(X * smooth_inv)."""
    lib = N.load()
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise ValueError("X must be a 2-D bf16 tensor")
    M, K = X.shape
    if smooth_inv is not None and (smooth_inv.dtype != torch.float32 or smooth_inv.numel() != K):
        raise ValueError("smooth_inv must be float32 [K]")
    if scale is None:
        scale = torch.empty(2, dtype=torch.float32, device=X.device)
    if scale.dtype != torch.float32 or scale.numel() < 2:
        raise ValueError("scale must be float32 [2]")
    N.check(lib.svdq_tensor_scale(M, K, _ptr(X), X.stride(0), _ptr(smooth_inv), _ptr(scale),
                                  _stream(stream)), "svdq_tensor_scale")
    return scale


def svdq_quantize_act_two_level(X: torch.Tensor, scale: torch.Tensor, L1s: torch.Tensor | None = None,
                                smooth_inv: torch.Tensor | None = None,
                                codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                                xl1: torch.Tensor | None = None, stream=None):
    """svdq_quantize_act in two-level NVFP4: codes and group scales of RN32(x_hat * scale[1]);
    ``scale`` is the float32 [2] pair from svdq_tensor_scale. Returns (codes, scales, xl1)."""
    lib = N.load()
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise ValueError("X must be a 2-D bf16 tensor")
    if scale.dtype != torch.float32 or scale.numel() < 2:
        raise ValueError("scale must be float32 [2]")
    M, K = X.shape
    r = 0 if L1s is None else L1s.shape[1]
    f = N.NVFP4_G16
    dev = X.device
    if codes is None:
        codes = torch.empty(lib.svdq_codes_bytes(f, M, K), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(lib.svdq_scales_bytes(f, M, K), dtype=torch.uint8, device=dev)
    S = lib.svdq_xl1_splits(M, K, r) if r else 0
    if r and xl1 is None:
        xl1 = torch.empty((S, M, r), dtype=torch.float32, device=dev)
    _need(codes, lib.svdq_codes_bytes(f, M, K), "codes")
    _need(scales, lib.svdq_scales_bytes(f, M, K), "scales")
    if L1s is not None and (L1s.dtype != torch.bfloat16 or tuple(L1s.shape) != (2, r, K)):
        raise ValueError("L1s must be bf16 [2, r, K]")
    if smooth_inv is not None and (smooth_inv.dtype != torch.float32 or smooth_inv.numel() != K):
        raise ValueError("smooth_inv must be float32 [K]")
    if xl1 is not None and (xl1.dtype != torch.float32 or xl1.numel() < S * M * r):
        raise ValueError(f"xl1 must be float32 [{S}, M, r]")
    N.check(lib.svdq_quantize_act_two_level(M, K, r, _ptr(X), K, _ptr(smooth_inv), _ptr(scale),
                                            _ptr(L1s), _ptr(codes), _ptr(scales),
                                            _ptr(xl1) if r else None, _stream(stream)),
            "svdq_quantize_act_two_level")
    return codes, scales, (xl1.view(-1)[:M * r].view(M, r) if r else None)


def svdq_w4a4_linear_two_level(a_codes, a_scales, a_tscale, xl1, w_codes, w_scales, w_tscale, L2,
                               bias, M: int, N_: int, K: int, out_dtype=torch.bfloat16,
                               Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Two-level NVFP4 W4A4 linear: Y = RN32(s_a s_w) * (4-bit product) + xl1 @ L2 + bias, with
    a_tscale / w_tscale the float32 scale pairs of the activation and the weight."""
    lib = N.load()
    r = 0 if L2 is None else L2.shape[0]
    if r and (xl1 is None or xl1.dtype != torch.float32 or xl1.numel() < M * r):
        raise ValueError("xl1 must be float32 [M, r]")
    for name, t in (("a_tscale", a_tscale), ("w_tscale", w_tscale)):
        if t is None or t.dtype != torch.float32 or t.numel() < 1:
            raise ValueError(f"{name} must be a float32 tensor scale pair")
    out = N.OUT_F32 if out_dtype == torch.float32 else N.OUT_BF16
    if Y is None:
        Y = torch.empty((M, N_), dtype=out_dtype, device=a_codes.device)
    if Y.dtype != out_dtype or Y.dim() != 2 or Y.shape[0] != M or Y.shape[1] < N_:
        raise ValueError("Y must be [M, >= N] of out_dtype")
    if L2 is not None and (L2.dtype != torch.bfloat16 or tuple(L2.shape) != (r, N_)):
        raise ValueError("L2 must be bf16 [r, N]")
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != N_):
        raise ValueError("bias must be bf16 [N]")
    f = N.NVFP4_G16
    _need(a_codes, lib.svdq_codes_bytes(f, M, K), "a_codes")
    _need(a_scales, lib.svdq_scales_bytes(f, M, K), "a_scales")
    _need(w_codes, lib.svdq_codes_bytes(f, N_, K), "w_codes")
    _need(w_scales, lib.svdq_scales_bytes(f, N_, K), "w_scales")
    N.check(lib.svdq_w4a4_linear_two_level(M, N_, K, r, _ptr(a_codes), _ptr(a_scales), _ptr(a_tscale),
                                           _ptr(xl1) if r else None, _ptr(w_codes), _ptr(w_scales),
                                           _ptr(w_tscale), _ptr(L2) if r else None, _ptr(bias),
                                           _ptr(Y), Y.shape[1], out, _stream(stream)),
            "svdq_w4a4_linear_two_level")
    return Y


def awq_w4a16_linear(X: torch.Tensor, qweight: torch.Tensor, sz: torch.Tensor,
                     bias: torch.Tensor | None, N_: int, group: int = 64,
                     Y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Step a7: Y [M, N] bf16 from X [M, K] bf16 and packed AWQ weights."""
    lib = N.load()
    if X.dtype != torch.bfloat16 or X.dim() != 2:
        raise ValueError("X must be a 2-D bf16 tensor")
    M, K = X.shape
    if Y is None:
        Y = torch.empty((M, N_), dtype=torch.bfloat16, device=X.device)
    _need(qweight, lib.awq_qweight_bytes(N_, K), "qweight")
    _need(sz, lib.awq_sz_bytes(N_, K), "sz")
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.numel() != N_):
        raise ValueError("bias must be bf16 [N]")
    N.check(lib.awq_w4a16_linear(M, N_, K, group, _ptr(X), _ptr(qweight), _ptr(sz), _ptr(bias),
                                 _ptr(Y), _stream(stream)), "awq_w4a16_linear")
    return Y


def svdq_column_absmax(A: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """absmax [K] float32 = max over rows of |A| for a 2-D bf16 tensor A [rows, K]."""
    lib = N.load()
    if A.dtype != torch.bfloat16 or A.dim() != 2:
        raise ValueError("A must be a 2-D bf16 tensor")
    rows, K = A.shape
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=A.device)
    if out.dtype != torch.float32 or out.numel() != K:
        raise ValueError("out must be float32 [K]")
    N.check(lib.svdq_column_absmax(rows, K, _ptr(A), K, _ptr(out), _stream(stream)), "svdq_column_absmax")
    return out


def svdq_smoothing(x_absmax: torch.Tensor, W: torch.Tensor, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """smooth_inv [K] float32 = RN32(1 / lambda), lambda = sqrt(x_absmax / max_n |W[n]|)
    in float64 (1 where either maximum is 0)."""
    lib = N.load()
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise ValueError("W must be a 2-D bf16 tensor")
    Nr, K = W.shape
    if x_absmax.dtype != torch.float32 or x_absmax.numel() != K:
        raise ValueError("x_absmax must be float32 [K]")
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=W.device)
    N.check(lib.svdq_smoothing(Nr, K, _ptr(x_absmax), _ptr(W), _ptr(out), _stream(stream)), "svdq_smoothing")
    return out


def svdq_lowrank_factors(U: torch.Tensor, S: torch.Tensor, Vh: torch.Tensor, r: int, stream=None):
    """(L1 [K, r], L2 [r, N]) bf16 from the float64 SVD W_hat = U diag(S) Vh, each element
    rounded once: L1 = RN_bf16(Vh[:r]^T sqrt(S_r)), L2 = RN_bf16(sqrt(S_r) U[:, :r]^T)."""
    lib = N.load()
    if U.dtype != torch.float64 or S.dtype != torch.float64 or Vh.dtype != torch.float64:
        raise ValueError("U, S, Vh must be float64")
    U, S, Vh = U.contiguous(), S.contiguous(), Vh.contiguous()
    Nr, K = U.shape[0], Vh.shape[1]
    L1 = torch.empty((K, r), dtype=torch.bfloat16, device=U.device)
    L2 = torch.empty((r, Nr), dtype=torch.bfloat16, device=U.device)
    N.check(lib.svdq_lowrank_factors(Nr, K, r, _ptr(U), U.shape[1], _ptr(S), _ptr(Vh), K, _ptr(L1),
                                     _ptr(L2), _stream(stream)), "svdq_lowrank_factors")
    return L1, L2


def svdq_residual(W: torch.Tensor, smooth_inv: torch.Tensor, L1: torch.Tensor | None,
                  L2: torch.Tensor | None, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """R [N, K] bf16 = RN_bf16(W diag(1 / smooth_inv) - (L1 L2)^T), float64 inside."""
    lib = N.load()
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise ValueError("W must be a 2-D bf16 tensor")
    Nr, K = W.shape
    r = 0 if L1 is None else L1.shape[1]
    if r and (L1.dtype != torch.bfloat16 or tuple(L1.shape) != (K, r) or L2 is None
              or L2.dtype != torch.bfloat16 or tuple(L2.shape) != (r, Nr)):
        raise ValueError("L1 must be bf16 [K, r] and L2 bf16 [r, N]")
    if smooth_inv.dtype != torch.float32 or smooth_inv.numel() != K:
        raise ValueError("smooth_inv must be float32 [K]")
    if out is None:
        out = torch.empty((Nr, K), dtype=torch.bfloat16, device=W.device)
    N.check(lib.svdq_residual(Nr, K, r, _ptr(W), _ptr(smooth_inv), _ptr(L1), _ptr(L2) if r else None,
                              _ptr(out), _stream(stream)), "svdq_residual")
    return out


def awq_quantize_weight(W: torch.Tensor, stream=None):
    """The AWQ int4 g64 quantizer of W [N, K] bf16, straight into the tiled layouts
    awq_w4a16_linear reads. Returns (qweight, sz) as uint8 tensors."""
    lib = N.load()
    if W.dtype != torch.bfloat16 or W.dim() != 2:
        raise ValueError("W must be a 2-D bf16 tensor")
    Nr, K = W.shape
    qt = torch.empty(lib.awq_qweight_bytes(Nr, K), dtype=torch.uint8, device=W.device)
    szt = torch.empty(lib.awq_sz_bytes(Nr, K), dtype=torch.uint8, device=W.device)
    N.check(lib.awq_quantize_weight(Nr, K, _ptr(W), _ptr(qt), _ptr(szt), _stream(stream)),
            "awq_quantize_weight")
    return qt, szt


def svdq_pack(kind, fmt, rows: int, K: int, plain_codes, plain_scales, plain_zeros=None,
              tiled_codes=None, tiled_scales=None, stream=None):
    """Plain -> tiled storage. Returns (tiled_codes, tiled_scales) as uint8 tensors."""
    lib = N.load()
    k = PACK_KINDS[kind] if isinstance(kind, str) else int(kind)
    f = _fmt(fmt)
    dev = plain_codes.device
    if k == N.PACK_AWQ:
        nc, ns = lib.awq_qweight_bytes(rows, K), lib.awq_sz_bytes(rows, K)
    else:
        nc, ns = lib.svdq_codes_bytes(f, rows, K), lib.svdq_scales_bytes(f, rows, K)
    if tiled_codes is None:
        tiled_codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    if tiled_scales is None:
        tiled_scales = torch.empty(ns, dtype=torch.uint8, device=dev)
    _need(tiled_codes, nc, "tiled_codes")
    _need(tiled_scales, ns, "tiled_scales")
    N.check(lib.svdq_pack(k, f, rows, K, _ptr(plain_codes), _ptr(plain_scales), _ptr(plain_zeros),
                          _ptr(tiled_codes), _ptr(tiled_scales), _stream(stream)), "svdq_pack")
    return tiled_codes, tiled_scales


def svdq_unpack(kind, fmt, rows: int, K: int, tiled_codes, tiled_scales, plain_codes,
                plain_scales, plain_zeros=None, stream=None):
    """Tiled -> plain storage, into caller-provided tensors."""
    lib = N.load()
    k = PACK_KINDS[kind] if isinstance(kind, str) else int(kind)
    N.check(lib.svdq_unpack(k, _fmt(fmt), rows, K, _ptr(tiled_codes), _ptr(tiled_scales),
                            _ptr(plain_codes), _ptr(plain_scales), _ptr(plain_zeros),
                            _stream(stream)), "svdq_unpack")
    return plain_codes, plain_scales, plain_zeros


def svdq_check_device_status(stream=None) -> int:
    """Synchronise the stream; return the status code (and clear the word)."""
    return N.load().svdq_check_device_status(_stream(stream))


def svdq_debug_wait_timeout(limit_us: int, stream=None) -> None:
    N.check(N.load().svdq_debug_wait_timeout(limit_us, _stream(stream)), "svdq_debug_wait_timeout")
