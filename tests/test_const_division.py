"""The quantizer's division of a group's absolute maximum by 6 (NVFP4) or 7
(INT4) is one multiply by c = RN32(1/b), an exact FMA remainder and one FMA
correction (Markstein's correction step for a known divisor). This restates
those float32 steps on the CPU and checks, for every float32 mantissa of the
binades the E4M3 and FP16 scale ranges reach (and a few beyond), that they
give the IEEE quotient -- so the scale codes stay bit-exact against the
oracle's RN32(amax / b). CPU only; no oracle code is involved."""

from fractions import Fraction

import numpy as np
import pytest

C_BITS = {6: 0x3E2AAAAB, 7: 0x3E124925}


def _f32(bits: int) -> np.float32:
    return np.array([bits], dtype=np.uint32).view(np.float32)[0]


def _method(a: np.ndarray, b: int) -> np.ndarray:
    c = _f32(C_BITS[b])
    q0 = a * c                                                   # RN32(a c)
    rem64 = a.astype(np.float64) - q0.astype(np.float64) * b    # exact in float64
    rem = rem64.astype(np.float32)
    assert np.array_equal(rem.astype(np.float64), rem64), "the FMA remainder must be exact"
    # RN32(q0 + rem c) with one rounding: rem c is exact in float64; the sum
    # may round there, so values next to a float32 midpoint are redone exactly
    s = q0.astype(np.float64) + rem.astype(np.float64) * np.float64(c)
    q = s.astype(np.float32)
    half = 0.5 * np.spacing(q).astype(np.float64)
    near = np.nonzero(np.abs(np.abs(s - q.astype(np.float64)) - half) <= np.abs(s) * 2.0 ** -45)[0]
    for j in near:
        exact = Fraction(float(q0[j])) + Fraction(float(rem[j])) * Fraction(float(c))
        lo = np.float32(float(exact))
        cands = [np.nextafter(lo, np.float32(-np.inf)), lo, np.nextafter(lo, np.float32(np.inf))]
        q[j] = min(cands, key=lambda v: (abs(Fraction(float(v)) - exact),
                                         int(np.array(v).view(np.uint32)) & 1))
    return q


def test_reciprocal_constants_are_rounded_reciprocals():
    for b, bits in C_BITS.items():
        assert _f32(bits) == np.float32(1.0) / np.float32(b)


@pytest.mark.parametrize("b", [6, 7])
@pytest.mark.parametrize("e", [-24, -10, -1, 0, 8, 11, 60])
def test_correction_step_gives_the_ieee_quotient(b, e):
    i = np.arange(1 << 23, dtype=np.uint32)
    a = ((np.uint32(e + 127) << np.uint32(23)) | i).view(np.float32)
    q = _method(a, b)
    ref = a / np.float32(b)
    assert np.array_equal(q.view(np.uint32), ref.view(np.uint32))


def test_zero_and_underflow():
    for b in (6, 7):
        assert _method(np.zeros(1, np.float32), b)[0] == 0.0
        tiny = np.array([2.0 ** -120, 2.0 ** -100], dtype=np.float32)
        # quotients far below the smallest E4M3 (2^-9) and FP16 (2^-24) scales
        assert np.all(_method(tiny, b) < 2.0 ** -60)
