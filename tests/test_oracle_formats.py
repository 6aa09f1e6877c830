"""Pins for the oracle's number formats, against things other than the oracle:
hand-written tables from the format definitions (tests/golden), the
independent ml_dtypes conversions, and numpy's IEEE binary16."""

import os

import ml_dtypes
import numpy as np
import pytest

from oracle import formats as F

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _read_table(path):
    rows = []
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            a, b = line.split()
            rows.append((float(a), int(b, 16)))
    return rows


def test_e2m1_golden_table(golden_dir):
    rows = _read_table(os.path.join(golden_dir, "e2m1_rne.txt"))
    x = np.array([r[0] for r in rows])
    want = np.array([r[1] for r in rows], dtype=np.uint8)
    got = F.e2m1_encode(x)
    assert np.array_equal(got, want), list(zip(x, got, want))


def test_ue4m3_golden_table(golden_dir):
    rows = _read_table(os.path.join(golden_dir, "ue4m3_points.txt"))
    x = np.array([r[0] for r in rows])
    want = np.array([r[1] for r in rows], dtype=np.uint8)
    assert np.array_equal(F.ue4m3_encode(x), want)


def _f32_sweep(lo_exp, hi_exp):
    """Float32 values with every top-16 mantissa pattern and a few low-bit
    patterns, across a range of exponents: covers every grid tie and both of
    its float32 neighbours for E2M1 and E4M3."""
    e = np.arange(127 + lo_exp, 127 + hi_exp + 1, dtype=np.uint32)
    hi = np.arange(1 << 16, dtype=np.uint32) << 7
    lo = np.array([0, 1, 0x3F, 0x40, 0x41, 0x7F], dtype=np.uint32)
    bits = (e[:, None, None] << 23) | hi[None, :, None] | lo[None, None, :]
    v = bits.reshape(-1).view(np.float32).astype(np.float64)
    return np.concatenate([v, [0.0]])


def test_e2m1_matches_ml_dtypes_exhaustively():
    v = _f32_sweep(-4, 2)          # 2^-4 .. 8: every tie of the E2M1 grid
    v = np.concatenate([v, -v])
    ours = F.e2m1_encode(v)
    theirs = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(ours, theirs)
    # decoded values agree as well
    assert np.array_equal(F.e2m1_decode(ours), v.astype(ml_dtypes.float4_e2m1fn).astype(np.float64))


def test_e2m1_is_nearest_with_even_ties():
    """Property: the chosen grid value is a nearest one; on a tie the code is even."""
    v = np.abs(_f32_sweep(-4, 2))
    v = v[v <= 6.0]
    code = F.e2m1_encode(v) & 7
    got = F.E2M1_MAGNITUDES[code]
    dist = np.abs(F.E2M1_MAGNITUDES[None, :] - v[:, None])
    best = dist.min(axis=1)
    assert np.all(np.abs(got - v) == best)
    ties = (dist == best[:, None]).sum(axis=1) > 1
    assert np.all(code[ties] % 2 == 0)


def test_ue4m3_matches_ml_dtypes_and_torch():
    import torch
    v = _f32_sweep(-12, 8)
    v = v[v <= 448.0]
    ours = F.ue4m3_encode(v)
    theirs = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, theirs)
    t = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, t)


def test_ue4m3_saturates_and_decodes():
    assert F.ue4m3_encode(np.array([448.0, 449.0, 463.9, 464.0, 1e9])).tolist() == [0x7E] * 5
    assert F.ue4m3_decode(np.array([0x7E]))[0] == 448.0
    assert F.ue4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert F.ue4m3_decode(np.array([0x08]))[0] == 2.0 ** -6
    with pytest.raises(ValueError):
        F.ue4m3_decode(np.array([0x7F]))


def test_fp16_round_closed_forms():
    one = 1.0
    ulp = 2.0 ** -10
    assert F.fp16_round(one + ulp / 2) == one                 # tie to even mantissa
    assert F.fp16_round(one + 3 * ulp / 2) == one + 2 * ulp   # tie to even, upward
    assert F.fp16_round(one + ulp / 2 + 2.0 ** -20) == one + ulp
    assert F.fp16_round(2.0 ** -24) == 2.0 ** -24             # smallest subnormal
    assert F.fp16_round(2.0 ** -25) == 0.0                    # half of it: tie to 0
    assert F.fp16_round(65504.0) == 65504.0


def test_bf16_round_single_rounding():
    rng = np.random.default_rng(3)
    v32 = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    # on float32 inputs one rounding equals ml_dtypes' conversion
    assert np.array_equal(F.bf16_round(v32.astype(np.float64)),
                          v32.astype(ml_dtypes.bfloat16).astype(np.float64))
    # a float64 input just above a bf16 half-way point rounds up, although its
    # float32 neighbour is exactly the half-way point
    x = float.fromhex("0x1.790000c328205p-7")
    assert F.bf16_round(np.array([x]))[0] == float.fromhex("0x1.7ap-7")
    assert F.bf16_round(np.array([float.fromhex("0x1.79p-7")]))[0] == float.fromhex("0x1.78p-7")


def test_rn32_is_float32_rounding():
    assert F.rn32(1.0 + 2.0 ** -24) == 1.0
    assert F.rn32(1.0 + 3 * 2.0 ** -24) == 1.0 + 2.0 ** -22
    assert F.rn32(1.0 / 3.0) == float(np.float32(1.0) / np.float32(3.0))
