"""User-facing layers over the C ABI: the SVDQ W4A4 linear and the AWQ W4A16
linear (the ``SVDQW4A4Linear`` / ``AWQW4A16Linear`` runtime layers of the
Diffusers blog, "quantization_config"), with preallocated workspaces so a
forward call is two (or one) library calls and no allocation."""

from __future__ import annotations

import torch

from . import prep
from . import (awq_w4a16_linear, svdq_codes_bytes, svdq_quantize_act, svdq_quantize_act_two_level,
               svdq_scales_bytes, svdq_tensor_scale, svdq_w4a4_linear, svdq_w4a4_linear_qkv_norm_rope,
               svdq_w4a4_linear_two_level, svdq_xl1_splits)


class SvdqW4A4Linear:
    """Y = Q(X_hat) Q(R)^T + (X_hat L1) L2 + bias on prepared weights.

    Weights prepared with a per-tensor scale (``w_tscale``) make the layer two-level
    NVFP4: the activation's scale pair is ``act_scale`` (float32 [2], calibrated) or,
    when that is None, computed on the device for every call."""

    def __init__(self, weights: dict, bias: torch.Tensor | None, max_tokens: int,
                 act_scale: torch.Tensor | None = None):
        self.w = weights
        self.bias = bias
        self.two_level = weights.get("w_tscale") is not None
        self.act_scale = act_scale
        self._a_scale = (torch.empty(2, dtype=torch.float32, device=weights["w_codes"].device)
                         if self.two_level else None)
        self.fmt = weights["fmt"]
        self.N, self.K, self.r = weights["N"], weights["K"], weights["r"]
        dev = weights["w_codes"].device
        self.max_tokens = max_tokens
        self.codes = torch.empty(svdq_codes_bytes(self.fmt, max_tokens, self.K), dtype=torch.uint8,
                                 device=dev)
        self.scales = torch.empty(svdq_scales_bytes(self.fmt, max_tokens, self.K), dtype=torch.uint8,
                                  device=dev)
        # the down-projection's partial sums: at most 8 splits of max_tokens rows
        self.xl1 = (torch.empty(8 * max_tokens * self.r, dtype=torch.float32, device=dev)
                    if self.r else None)

    @classmethod
    def from_linear(cls, weight: torch.Tensor, bias: torch.Tensor | None, x_absmax: torch.Tensor,
                    rank: int, max_tokens: int, fmt: str = "nvfp4", two_level: bool = False,
                    act_scale: torch.Tensor | None = None):
        """From an nn.Linear's weight [N, K] bf16 (and bias [N] bf16 or None) and the
        calibration activations' per-channel max |X| [K]: smoothing, SVD split and the
        residual quantized by the library (prep.prepare_svdq_weights)."""
        w = prep.prepare_svdq_weights(weight, x_absmax, rank, fmt, two_level=two_level)
        return cls(w, bias, max_tokens, act_scale=act_scale)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        M = x.shape[0]
        if M > self.max_tokens:
            raise ValueError(f"{M} tokens > workspace for {self.max_tokens}")
        xl1 = self.xl1[:svdq_xl1_splits(M, self.K, self.r) * M * self.r] if self.r else None
        if self.two_level:
            a_scale = self.act_scale
            if a_scale is None:
                a_scale = svdq_tensor_scale(x, self.w["smooth_inv"], self._a_scale, stream=stream)
            codes, scales, xl1 = svdq_quantize_act_two_level(
                x, a_scale, self.w["L1s"], self.w["smooth_inv"], codes=self.codes, scales=self.scales,
                xl1=xl1, stream=stream)
            return svdq_w4a4_linear_two_level(codes, scales, a_scale, xl1, self.w["w_codes"],
                                              self.w["w_scales"], self.w["w_tscale"], self.w["L2"],
                                              self.bias, M, self.N, self.K, Y=y, stream=stream)
        codes, scales, xl1 = svdq_quantize_act(x, self.w["L1s"], self.w["smooth_inv"], fmt=self.fmt,
                                               codes=self.codes, scales=self.scales, xl1=xl1,
                                               stream=stream)
        return svdq_w4a4_linear(codes, scales, xl1, self.w["w_codes"], self.w["w_scales"], self.w["L2"],
                                self.bias, M, self.N, self.K, fmt=self.fmt, Y=y, stream=stream)

    __call__ = forward


class SvdqQkvNormRope(SvdqW4A4Linear):
    """The fused QKV projection of an attention block (Diffusers blog, the fused QKV
    section: to_q, to_k, to_v joined into one SVDQ linear, followed by norm_q / norm_k
    per head and the rotary embedding in one fused call). Weights prepared for the
    joined [3 H 128, K] projection, NVFP4, one-level; norm_q, norm_k bf16 [128] or None.
    forward(x, rope_cos, rope_sin) takes the rows' angle tables, float32 [64, M] each,
    angle-major (or None: no rotation), and returns Q | K | V [M, 3 H 128], Q and K
    normalised and rotated."""

    def __init__(self, weights: dict, bias: torch.Tensor | None, max_tokens: int,
                 norm_q: torch.Tensor | None = None, norm_k: torch.Tensor | None = None,
                 eps: float = 1e-6):
        if weights["fmt"] != "nvfp4" or weights.get("w_tscale") is not None:
            raise ValueError("the fused QKV projection takes one-level NVFP4 weights")
        if weights["N"] % 384:
            raise ValueError(f"N = {weights['N']} is not Q, K, V of whole 128-column heads")
        super().__init__(weights, bias, max_tokens)
        self.norm_q, self.norm_k, self.eps = norm_q, norm_k, float(eps)
        self.heads = weights["N"] // 384

    @classmethod
    def from_linears(cls, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                     biases: tuple | None, x_absmax: torch.Tensor, rank: int, max_tokens: int,
                     norm_q: torch.Tensor | None = None, norm_k: torch.Tensor | None = None,
                     eps: float = 1e-6):
        """From the to_q, to_k, to_v weights [H 128, K] bf16 (biases: three [H 128] bf16
        tensors or None each, or None): the three are joined along the output dimension
        in the order Q, K, V into one [3 H 128, K] projection, which is prepared once
        (smoothing from x_absmax, SVD split, quantized residual)."""
        if not (q.shape == k.shape == v.shape) or q.dim() != 2 or q.shape[0] % 128:
            raise ValueError("to_q, to_k, to_v must be equal [H 128, K] weights")
        w = torch.cat([q, k, v], dim=0)
        bias = None
        if biases is not None and any(b is not None for b in biases):
            bias = torch.cat([b if b is not None else torch.zeros(q.shape[0], dtype=q.dtype, device=q.device)
                              for b in biases])
        return cls.from_linear(w, bias, x_absmax, rank, max_tokens, norm_q=norm_q, norm_k=norm_k, eps=eps)

    @classmethod
    def from_linear(cls, weight: torch.Tensor, bias: torch.Tensor | None, x_absmax: torch.Tensor,
                    rank: int, max_tokens: int, norm_q: torch.Tensor | None = None,
                    norm_k: torch.Tensor | None = None, eps: float = 1e-6):
        """From an already joined to_qkv weight [3 H 128, K] bf16 (rows Q, then K, then V)."""
        weights = prep.prepare_svdq_weights(weight, x_absmax, rank, "nvfp4")
        return cls(weights, bias, max_tokens, norm_q=norm_q, norm_k=norm_k, eps=eps)

    def forward(self, x: torch.Tensor, rope_cos: torch.Tensor | None = None,
                rope_sin: torch.Tensor | None = None, y: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
        M = x.shape[0]
        if M > self.max_tokens:
            raise ValueError(f"{M} tokens > workspace for {self.max_tokens}")
        xl1 = self.xl1[:svdq_xl1_splits(M, self.K, self.r) * M * self.r] if self.r else None
        codes, scales, xl1 = svdq_quantize_act(x, self.w["L1s"], self.w["smooth_inv"], fmt="nvfp4",
                                               codes=self.codes, scales=self.scales, xl1=xl1,
                                               stream=stream)
        return svdq_w4a4_linear_qkv_norm_rope(codes, scales, xl1, self.w["w_codes"], self.w["w_scales"],
                                              self.w["L2"], self.bias, self.norm_q, self.norm_k,
                                              rope_cos, rope_sin, M, self.N, self.K, eps=self.eps, Y=y,
                                              stream=stream)

    __call__ = forward


class AwqW4A16Linear:
    def __init__(self, weights: dict, bias: torch.Tensor | None):
        self.w = weights
        self.bias = bias

    @classmethod
    def from_linear(cls, weight: torch.Tensor, bias: torch.Tensor | None):
        """From an nn.Linear's weight [N, K] bf16: asymmetric int4, group 64, packed
        (prep.prepare_awq_weights)."""
        return cls(prep.prepare_awq_weights(weight), bias)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        return awq_w4a16_linear(x, self.w["qweight"], self.w["sz"], self.bias, self.w["N"], Y=y,
                                stream=stream)

    __call__ = forward
