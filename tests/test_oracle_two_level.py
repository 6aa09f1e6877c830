"""Pins of the oracle's two-level NVFP4 (a per-tensor float32 scale above the
E4M3 group scales), against facts that do not restate its formulas: exact
power-of-two scaling, the identity case, the error the format must reach on
tensors whose range E4M3 group scales alone cannot cover, and the unquantized
product the layer approximates."""

import numpy as np
import pytest

from oracle import svdq as S

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def f32(a):
    return np.asarray(a, np.float32).astype(np.float64)


def in_range_tensor(rng, shape):
    """Float32 values whose absolute maximum is exactly 6 * 448 (tensor scale 1)."""
    y = f32(rng.standard_normal(shape))
    y = f32(y / np.max(np.abs(y)) * 2000.0)
    y.flat[int(np.argmax(np.abs(y)))] = 2688.0
    return y


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_tensor_scale_closed_forms():
    assert S.tensor_scale(np.array([[2688.0, -3.0]])) == (1.0, 1.0)
    assert S.tensor_scale(np.zeros((4, 16))) == (1.0, 1.0)
    for k in (-40, -9, 1, 30, 100):
        s, inv = S.tensor_scale(np.array([[-2688.0 * 2.0 ** k, 1000.0 * 2.0 ** k]]))
        assert (s, inv) == (2.0 ** k, 2.0 ** -k)
    # a quotient that underflows to a subnormal falls back to 1
    assert S.tensor_scale(np.array([[1e-40]])) == (1.0, 1.0)
    # in general: s_t is the float32 nearest amax / 2688 and inv the float32 nearest 1 / s_t
    for amax in (1.0, 3.3e-5, 7.1e8):
        s, inv = S.tensor_scale(np.array([[amax]]))
        assert abs(s * 2688.0 - f32(amax)) <= 2.0 ** -24 * f32(amax)
        assert abs(s * inv - 1.0) <= 2.0 ** -24


def test_scale_one_is_the_one_level_format():
    y = in_range_tensor(np.random.default_rng(0), (8, 64))
    s, inv = S.tensor_scale(y)
    assert (s, inv) == (1.0, 1.0)
    q2, sc2 = S.quantize_nvfp4_two_level(y, inv)
    q1, sc1 = S.quantize_nvfp4(y)
    assert np.array_equal(q1, q2) and np.array_equal(sc1, sc2)


@pytest.mark.parametrize("k", [-60, -12, 15, 90])
def test_power_of_two_tensors_scale_exactly(k):
    """x = y 2^k quantizes to y's codes and scales, and dequantizes to exactly 2^k times y's."""
    y = in_range_tensor(np.random.default_rng(1 + k % 7), (6, 128))
    x = y * 2.0 ** k
    s, inv = S.tensor_scale(x)
    assert s == 2.0 ** k
    q, sc = S.quantize_nvfp4_two_level(x, inv)
    qy, scy = S.quantize_nvfp4(y)
    assert np.array_equal(q, qy) and np.array_equal(sc, scy)
    assert np.array_equal(S.dequant_nvfp4_two_level(q, sc, s), S.dequant_nvfp4(qy, scy) * 2.0 ** k)


@pytest.mark.parametrize("magnitude", [3e6, 1e-8])
def test_two_level_covers_what_group_scales_alone_cannot(magnitude):
    """Far outside E4M3's range one level saturates (or underflows to zero) while
    two levels keep the format's relative error (a few percent on Gaussian data)."""
    x = f32(np.random.default_rng(2).standard_normal((16, 256)) * magnitude)
    q1, sc1 = S.quantize_nvfp4(x)
    err1 = rel_l2(S.dequant_nvfp4(q1, sc1), x)
    s, inv = S.tensor_scale(x)
    q2, sc2 = S.quantize_nvfp4_two_level(x, inv)
    err2 = rel_l2(S.dequant_nvfp4_two_level(q2, sc2, s), x)
    assert err1 > 0.5
    assert err2 < 0.15


def test_layer_with_reciprocal_power_of_two_scales_equals_the_one_level_layer():
    """Activations scaled by 2^10 and weights by 2^-10: alpha = 1 and the two-level
    layer gives exactly the one-level layer of the unscaled tensors."""
    rng = np.random.default_rng(3)
    y, v = in_range_tensor(rng, (5, 64)), in_range_tensor(rng, (7, 64))
    xl1, L2, bias = f32(rng.standard_normal((5, 16))), f32(rng.standard_normal((16, 7))), f32(rng.standard_normal(7))
    x, w = y * 2.0 ** 10, v * 2.0 ** -10
    sa, inva = S.tensor_scale(x)
    sw, invw = S.tensor_scale(w)
    qa, sca = S.quantize_nvfp4_two_level(x, inva)
    qw, scw = S.quantize_nvfp4_two_level(w, invw)
    y2 = S.w4a4_linear_two_level(S.dequant_nvfp4(qa, sca), S.dequant_nvfp4(qw, scw), sa, sw, xl1, L2, bias)
    qy, scy = S.quantize_nvfp4(y)
    qv, scv = S.quantize_nvfp4(v)
    y1 = S.w4a4_linear(S.dequant_nvfp4(qy, scy), S.dequant_nvfp4(qv, scv), xl1, L2, bias)
    assert np.array_equal(y1, y2)


def test_two_level_layer_approximates_the_unquantized_product():
    """On tensors far out of E4M3's range the two-level layer stays within the
    format's error of x w^T + xl1 L2 + bias; the alpha factor is what carries the
    two tensor scales (dropping it would be off by about 1e12)."""
    rng = np.random.default_rng(4)
    x, w = f32(rng.standard_normal((12, 256)) * 4e6), f32(rng.standard_normal((24, 256)) * 2e-7)
    xl1, L2, bias = f32(rng.standard_normal((12, 16))), f32(rng.standard_normal((16, 24))), f32(rng.standard_normal(24))
    sa, inva = S.tensor_scale(x)
    sw, invw = S.tensor_scale(w)
    qa, sca = S.quantize_nvfp4_two_level(x, inva)
    qw, scw = S.quantize_nvfp4_two_level(w, invw)
    got = S.w4a4_linear_two_level(S.dequant_nvfp4(qa, sca), S.dequant_nvfp4(qw, scw), sa, sw, xl1, L2, bias)
    want = x @ w.T + xl1 @ L2 + bias[None, :]
    assert rel_l2(got, want) < 0.15
