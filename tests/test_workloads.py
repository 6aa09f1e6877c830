"""The seeded input module: deterministic, correctly rounded, right structure."""

import ml_dtypes
import numpy as np

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
