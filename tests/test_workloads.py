"""The seeded input module: deterministic, correctly rounded, right structure."""

import ml_dtypes
import numpy as np
import pytest

import workloads as WL


def test_bf16_rounding_matches_ml_dtypes_on_float32():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(100000) * np.exp(rng.uniform(-40, 40, 100000))).astype(np.float32)
    ours = WL.f32_to_bf16_bits(v)
    theirs = v.astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(ours, theirs)
    assert np.array_equal(WL.bf16_bits_to_f32(ours), v.astype(ml_dtypes.bfloat16).astype(np.float32))


def test_draws_are_deterministic_and_shaped():
    a = WL.svdq_inputs(WL.TINY)
    b = WL.svdq_inputs(WL.TINY)
    for k in ("X", "W", "bias"):
        assert np.array_equal(a[k], b[k])
    assert a["X"].shape == (256, 512) and a["W"].shape == (512, 512) and a["bias"].shape == (512,)
    x = WL.bf16_bits_to_f32(a["X"])
    col = np.abs(x).max(0)
    assert (col > 20).sum() == 4          # four outlier channels scaled by 30
    sub = WL.svdq_inputs(WL.TINY, M=100)
    assert np.array_equal(sub["X"], a["X"][:100])


def test_spike_is_present():
    shape = WL.custom_svdq("s", 8, 256, 192, 16, spike_rank=8, spike_sv=5.0)
    w = WL.bf16_bits_to_f32(WL.svdq_inputs(shape)["W"]).astype(np.float64)
    s = np.linalg.svd(w, compute_uv=False)
    assert np.all(s[:8] > 4.5) and s[8] < 0.02 * (np.sqrt(192) + np.sqrt(256)) * 1.2


def test_qkv_epilogue_inputs():
    a = WL.qkv_epilogue_inputs(37, seed=3)
    b = WL.qkv_epilogue_inputs(37, seed=3)
    assert all(np.array_equal(a[k], b[k]) for k in a)
    assert a["norm_q"].shape == (128,) and a["norm_q"].dtype == np.uint16
    assert a["cos"].shape == (37, 64) and a["cos"].dtype == np.float32
    # each (cos, sin) pair is a unit vector up to float32 rounding
    assert np.allclose(a["cos"].astype(np.float64) ** 2 + a["sin"].astype(np.float64) ** 2, 1.0, atol=1e-6)
    # position angles: row 0 is the identity, and pair 0 turns by exactly one radian per row
    p = WL.qkv_epilogue_inputs(5, seed=0, angles="positions")
    assert np.array_equal(p["cos"][0], np.ones(64, np.float32)) and not p["sin"][0].any()
    assert np.allclose(p["cos"][:, 0], np.cos(np.arange(5)), atol=1e-7)
    with pytest.raises(ValueError):
        WL.qkv_epilogue_inputs(5, seed=0, angles="random")
