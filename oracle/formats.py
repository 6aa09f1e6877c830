"""Number formats used by SVDQuant's 4-bit path, written out from their definitions.

ORACLE -- test infrastructure only. Nothing in the product package imports it.

All arithmetic here is float64 on values that are exactly representable in the
narrower format being modelled. ``rn32`` models one IEEE float32 operation:
float64 -> float32 round-to-nearest-even. For +, -, *, / and sqrt of float32
operands this double rounding (exact float64 op, then RN32) equals the single
float32 operation, because 53 >= 2*24 + 2.

Formats (the NVFP4 / INT4 precisions of the Diffusers blog, "quantization_config",
``precision: nvfp4, group_size: 16``; the Nunchaku README news on NVFP4 for
Blackwell):

* E2M1 (FP4): sign, 2 exponent bits (bias 1), 1 mantissa bit, no Inf/NaN.
  Magnitudes by code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Code bit 3 is the sign.
* UE4M3 (FP8 scale, unsigned use of E4M3): 4 exponent bits (bias 7), 3 mantissa
  bits, subnormals m * 2^-9, largest finite 448 (code 0x7E); 0x7F is NaN.
* FP16 (IEEE binary16) and BF16 (the top 16 bits of an IEEE float32).

Rounding is round-to-nearest, ties to the even code, with saturation to the
largest finite magnitude ("satfinite") for E2M1 and UE4M3.
"""

from __future__ import annotations

import numpy as np

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def rn32(x) -> np.ndarray:
    """One float32 rounding of a float64 value (IEEE round-to-nearest-even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def _ue4m3_table() -> np.ndarray:
    """Value of every finite non-negative E4M3 code, indexed by code 0..126."""
    vals = np.empty(127, dtype=np.float64)
    for c in range(127):
        e, m = c >> 3, c & 7
        if e == 0:
            vals[c] = m * 2.0 ** -9          # subnormal: 0.m * 2^(1-7)
        else:
            vals[c] = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


UE4M3_VALUES = _ue4m3_table()


def _round_to_grid(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the nearest grid point to each non-negative ``mag``.

    ``grid`` is sorted ascending and indexed by code, so "ties to even" means
    the tie goes to the even index. Magnitudes above the last point saturate
    to it.
    """
    mag = np.asarray(mag, dtype=np.float64)
    hi_cap = len(grid) - 1
    lo = np.searchsorted(grid, mag, side="right") - 1
    lo = np.clip(lo, 0, hi_cap)
    hi = np.minimum(lo + 1, hi_cap)
    d_lo = mag - grid[lo]
    d_hi = grid[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    idx = np.where(pick_hi, hi, lo)
    return np.where(mag >= grid[-1], hi_cap, idx)


def e2m1_encode(v) -> np.ndarray:
    """float64 -> 4-bit E2M1 code (uint8 0..15), RNE, satfinite, sign kept.

    A negative value whose magnitude rounds to zero keeps its sign (code 0x8),
    as an IEEE conversion of -x does.
    """
    v = np.asarray(v, dtype=np.float64)
    mag_code = _round_to_grid(np.abs(v), E2M1_MAGNITUDES).astype(np.uint8)
    sign = np.signbit(v).astype(np.uint8) << 3
    return (sign | mag_code).astype(np.uint8)


def e2m1_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where(codes & 8, -mag, mag)


def ue4m3_encode(v) -> np.ndarray:
    """float64 >= 0 -> E4M3 code (uint8 0..0x7E), RNE, satfinite at 448."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("ue4m3_encode takes non-negative finite values")
    return _round_to_grid(v, UE4M3_VALUES).astype(np.uint8)


def ue4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    if np.any(codes > 0x7E):
        raise ValueError("E4M3 code 0x7F is NaN; scales never use it")
    return UE4M3_VALUES[codes]


def fp16_round(v) -> np.ndarray:
    """float64 holding a float32 value -> nearest-even IEEE binary16, as float64."""
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float16).astype(np.float64)


def fp16_bits(v) -> np.ndarray:
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def fp16_from_bits(b) -> np.ndarray:
    return np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_from_bits(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_sig(v, bits: int) -> np.ndarray:
    """Round float64 values to ``bits`` significant bits, nearest-even.

    v = f * 2^e with 0.5 <= |f| < 1; scaling f by 2^bits is exact, rint rounds
    half-way cases to the even integer (the even mantissa), scaling back is exact.
    Only the normal range of the target format is modelled.
    """
    f, e = np.frexp(np.asarray(v, dtype=np.float64))
    return np.ldexp(np.rint(np.ldexp(f, bits)), e - bits)


def bf16_round(v) -> np.ndarray:
    """float64 -> nearest-even bfloat16 value (8 significant bits), one rounding."""
    return round_sig(v, 8)


def bf16_bits(v) -> np.ndarray:
    """Bit pattern of values that are already exact bfloat16 values."""
    f = np.ascontiguousarray(np.asarray(v, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("value is not a bfloat16 value")
    return (u >> 16).astype(np.uint16)
