"""Seeded synthetic inputs for the SVDQuant W4A4 linear and the AWQ W4A16 linear.

This module holds random draws and nothing else: no smoothing, no SVD, no
quantization. Both the CPU oracle (``oracle/``) and the CUDA path consume the
bytes it returns, so the two sides always see identical inputs.

Every tensor is drawn in float64 with ``numpy.random.default_rng(seed)``,
narrowed to float32 and then rounded to bfloat16 (round-to-nearest-even on
the float32 bits). Values are returned as uint16 bfloat16 bit patterns.

Distributions follow the layer shapes described for the SVDQuant engine
(Nunchaku README, "Method" and "Engine design"; the Diffusers blog,
"quantization_config" and the fused to_q/to_k/to_v projection):

* activations X [M, K] ~ N(0, 1), with ``n_outliers`` channels (picked by a
  seeded permutation of K) multiplied by ``outlier_scale``;
* weights W [N, K] ~ N(0, 0.02), optionally plus a rank-``spike_rank`` term
  U diag(spike_sv) V^T whose U and V are the Q factors of seeded Gaussian
  matrices (this is how one draws random orthonormal columns);
* bias [N] ~ N(0, 0.1).
"""

from __future__ import annotations

import dataclasses

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16, nearest-even, returning uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen uint16 bfloat16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64 draw -> float32 -> bfloat16 bits."""
    return f32_to_bf16_bits(np.asarray(a, dtype=np.float64).astype(np.float32))


@dataclasses.dataclass(frozen=True)
class SvdqShape:
    """One SVDQ W4A4 linear: Y[M,N] = X[M,K] W[N,K]^T (+ bias), rank r, format."""

    name: str
    M: int
    K: int
    N: int
    r: int
    fmt: str  # "nvfp4" (E2M1 + E4M3 scale per 16) or "int4" (symmetric, fp16 scale per 64)
    n_outliers: int
    outlier_scale: float
    spike_rank: int
    spike_sv: float
    bias: bool
    seed: int


@dataclasses.dataclass(frozen=True)
class AwqShape:
    """One AWQ W4A16 linear: Y[M,N] = X[M,K] dequant(W)[N,K]^T + bias, group 64."""

    name: str
    M: int
    K: int
    N: int
    group: int
    bias: bool
    seed: int


# The five workloads. Seeds are the workload index.
TINY = SvdqShape("tiny", 256, 512, 512, 16, "nvfp4", 4, 30.0, 0, 0.0, True, 0)
QKV = SvdqShape("flux_qkv", 4608, 3072, 9216, 32, "nvfp4", 16, 50.0, 8, 5.0, True, 1)
FC1 = SvdqShape("flux_fc1", 4608, 3072, 12288, 128, "nvfp4", 16, 50.0, 8, 5.0, True, 2)
FC2 = SvdqShape("flux_fc2", 4608, 12288, 3072, 128, "nvfp4", 16, 50.0, 8, 5.0, True, 102)
FC1_INT4 = SvdqShape("flux_fc1_int4", 4608, 3072, 12288, 128, "int4", 16, 50.0, 8, 5.0, True, 2)
RANK_SWEEP = [
    SvdqShape(f"dit3840_n{n}_r{r}", 4096, 3840, n, r, "nvfp4", 16, 50.0, 8, 5.0, True, 3)
    for n in (3840, 15360)
    for r in (0, 32, 128, 256)
]
BIG = SvdqShape("flux_qkv_b4", 18432, 3072, 9216, 32, "nvfp4", 16, 50.0, 8, 5.0, True, 4)
AWQ_MOD = AwqShape("adaln_mod_b4", 4, 3072, 18432, 64, True, 1004)

SVDQ_WORKLOADS = [TINY, QKV, FC1, FC2, FC1_INT4, *RANK_SWEEP, BIG]
ALL_WORKLOADS = {w.name: w for w in [*SVDQ_WORKLOADS, AWQ_MOD]}


def draw_activations(rng: np.random.Generator, M: int, K: int, n_outliers: int,
                     outlier_scale: float) -> np.ndarray:
    """X [M,K] ~ N(0,1) with n_outliers channels scaled up; bf16 bits."""
    x = rng.standard_normal((M, K))
    if n_outliers:
        idx = rng.permutation(K)[:n_outliers]
        x[:, idx] *= outlier_scale
    return to_bf16_bits(x)


def draw_weight(rng: np.random.Generator, N: int, K: int, std: float, spike_rank: int,
                spike_sv: float) -> np.ndarray:
    """W [N,K] ~ N(0,std) plus an optional rank-`spike_rank` spike; bf16 bits."""
    w = rng.standard_normal((N, K)) * std
    if spike_rank:
        u, _ = np.linalg.qr(rng.standard_normal((N, spike_rank)))
        v, _ = np.linalg.qr(rng.standard_normal((K, spike_rank)))
        w += (u * spike_sv) @ v.T
    return to_bf16_bits(w)


def draw_bias(rng: np.random.Generator, N: int) -> np.ndarray:
    return to_bf16_bits(rng.standard_normal(N) * 0.1)


def svdq_inputs(shape: SvdqShape, M: int | None = None) -> dict:
    """Draw X, W and bias for one SVDQ layer. ``M`` may shrink the row count
    (the first M rows of the full draw are returned, so a row sample of a
    full-size workload is the same bytes as the full workload's rows)."""
    rng = np.random.default_rng(shape.seed)
    x = draw_activations(rng, shape.M, shape.K, shape.n_outliers, shape.outlier_scale)
    w = draw_weight(rng, shape.N, shape.K, 0.02, shape.spike_rank, shape.spike_sv)
    b = draw_bias(rng, shape.N) if shape.bias else None
    if M is not None:
        x = x[:M].copy()
    return {"X": x, "W": w, "bias": b}


def awq_inputs(shape: AwqShape) -> dict:
    rng = np.random.default_rng(shape.seed)
    x = to_bf16_bits(rng.standard_normal((shape.M, shape.K)))
    w = to_bf16_bits(rng.standard_normal((shape.N, shape.K)) * 0.02)
    b = draw_bias(rng, shape.N) if shape.bias else None
    return {"X": x, "W": w, "bias": b}


def custom_svdq(name: str, M: int, K: int, N: int, r: int, fmt: str = "nvfp4",
                seed: int = 7, n_outliers: int = 4, outlier_scale: float = 30.0,
                spike_rank: int = 0, spike_sv: float = 0.0, bias: bool = True) -> SvdqShape:
    """A small workload of the same structure, for tests that need ragged sizes."""
    return SvdqShape(name, M, K, N, r, fmt, n_outliers, outlier_scale, spike_rank,
                     spike_sv, bias, seed)


def qkv_epilogue_inputs(M: int, seed: int, angles: str = "uniform") -> dict:
    """Inputs of the fused QKV epilogue: head weights gamma_q, gamma_k [128] as
    bfloat16 bits (~ 1 + N(0, 0.1), the spread of trained RMS-norm weights), and
    rotation tables cos, sin [M, 64] float32. ``angles`` "uniform" draws every
    angle from U(-pi, pi); "positions" takes row m as token position m with pair
    i at frequency 10000^(-i/64), the usual rotary layout of one position axis."""
    rng = np.random.default_rng(seed)
    gq = to_bf16_bits(1.0 + rng.standard_normal(128) * 0.1)
    gk = to_bf16_bits(1.0 + rng.standard_normal(128) * 0.1)
    if angles == "uniform":
        th = rng.uniform(-np.pi, np.pi, (M, 64))
    elif angles == "positions":
        th = np.arange(M, dtype=np.float64)[:, None] * 10000.0 ** (-np.arange(64) / 64.0)[None, :]
    else:
        raise ValueError(angles)
    return {"norm_q": gq, "norm_k": gk, "cos": np.cos(th).astype(np.float32),
            "sin": np.sin(th).astype(np.float32)}
