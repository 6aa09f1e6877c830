"""Shared helpers for tests: build one SVDQ layer with the oracle, move inputs to
the GPU, and compare results with the stated tolerances.

Oracle side: offline prep (smoothing, SVD split, residual quantization) and the
reference outputs. CUDA side: whatever the test calls through the binding.
"""

from __future__ import annotations

import numpy as np

import workloads as WL
from oracle import formats as F
from oracle import layout as LO
from oracle import prep as P
from oracle import svdq as S


def bf16_tensor(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def bf16_bits_of(t) -> np.ndarray:
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def u8_tensor(a: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device)


def f32_tensor(a: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def oracle_layer(shape: WL.SvdqShape, M: int | None = None) -> dict:
    """Inputs and oracle prep for one layer. X rows can be cut to M after prep
    (smoothing statistics always come from the full draw)."""
    d = WL.svdq_inputs(shape)
    pr = P.prepare_svdq_layer(shape.fmt, d["X"], d["W"], shape.r)
    x_bits = d["X"] if M is None else d["X"][:M].copy()
    return {"shape": shape, "x_bits": x_bits, "w_bits": d["W"], "bias_bits": d["bias"], **pr}


def tiled_codes(fmt: str, q: np.ndarray) -> np.ndarray:
    """Codes as the kernels store them: packed nibbles (INT4 two's complement)."""
    if fmt == "nvfp4":
        return S.pack_nibbles(q).reshape(-1)
    return LO.tile_int4_codes(q).reshape(-1)


def tiled_scales(fmt: str, scales: np.ndarray) -> np.ndarray:
    if fmt == "nvfp4":
        return LO.tile_nvfp4_scales(scales)
    return LO.tile_int4_scales(scales).view(np.uint8)


def rel_l2(y: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |v| (8 significant bits)."""
    _, e = np.frexp(np.abs(v))
    return np.ldexp(1.0, e - 9)


def assert_gemm_close(y: np.ndarray, ref: np.ndarray, bf16_out: bool, what: str = "Y"):
    """The stated pass criteria against the unrounded oracle: rel-L2 <= 2e-3 and
    max |err| <= 1e-2 rms(Y). For bf16 output the output's own rounding is added to
    both: half a bf16 ulp of the reference to the max-abs bound, and its relative
    size 2^-9 to the rel-L2 bound (|RN_bf16(y) - y| <= 2^-9 |y| per value, so a
    result whose float32 arithmetic meets 2e-3 stays within 2e-3 + 2^-9 once
    rounded; with only a few dozen outputs the rounding alone can come close to
    2^-9)."""
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(y - ref)
    rl = rel_l2(y, ref)
    rl_bound = 2e-3 + (2.0 ** -9 if bf16_out else 0.0)
    bound = 1e-2 * rms + (bf16_half_ulp(ref) if bf16_out else 0.0)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert rl <= rl_bound, f"{what}: rel-L2 {rl:.3e} > {rl_bound:.3e}"
    assert np.all(err <= bound), (
        f"{what}: max-abs check fails at {worst}: got {y[worst]}, want {ref[worst]}, "
        f"err {err[worst]:.3e}, bound {np.broadcast_to(bound, err.shape)[worst]:.3e}")
    return rl


def xl1_bound(xhat: np.ndarray, L1: np.ndarray) -> np.ndarray:
    """Error bound for the tensor-core down-projection: the bf16 hi/lo split of
    x_hat leaves at most 2^-16 relative per product, and float32 accumulation
    adds at most a few ulps of the running sum of |terms|."""
    absum = np.abs(xhat) @ np.abs(L1)
    return absum * (2.0 ** -16 + 64 * 2.0 ** -24) + 1e-30
