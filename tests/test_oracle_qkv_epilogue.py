"""Pins of the oracle's fused QKV epilogue (per-head RMS norm, then the pairwise
rotation) against facts that do not restate its formulas: the unit mean square
of a normalized head, exact invariance under power-of-two scaling, constant
heads, rotation as multiplication of complex numbers (numpy's complex
arithmetic), the quarter turn, composition of angles, and V left alone."""

import numpy as np
import pytest

from oracle import qkv_epilogue as E

D = E.HEAD_DIM


def heads(rng, M, H, scale=1.0):
    return rng.standard_normal((M, H, D)) * scale


def angles(rng, M):
    th = rng.uniform(-np.pi, np.pi, (M, D // 2))
    return th, np.cos(th), np.sin(th)


def test_normalized_head_has_unit_mean_square():
    v = heads(np.random.default_rng(0), 5, 3, 7.5)
    z = E.rms_norm_heads(v, None, 0.0)
    assert np.allclose(np.mean(z * z, axis=-1), 1.0, rtol=0, atol=1e-14)
    # the direction of each head is kept: z is a positive multiple of v
    ratio = z / v
    assert np.all(ratio > 0) and np.allclose(ratio, ratio[..., :1], rtol=1e-14)


@pytest.mark.parametrize("k", [-30, -3, 4, 25])
def test_power_of_two_scaling_leaves_the_norm_unchanged(k):
    v = heads(np.random.default_rng(1), 4, 2)
    g = np.random.default_rng(2).uniform(0.5, 2.0, D)
    assert np.array_equal(E.rms_norm_heads(v * 2.0 ** k, g, 0.0), E.rms_norm_heads(v, g, 0.0))


def test_constant_head_and_eps():
    # a head of equal values c has mean square c^2: the norm gives sign(c) gamma / sqrt(1 + eps / c^2)
    g = np.linspace(0.5, 1.5, D)
    v = np.full((1, 1, D), -3.0)
    assert np.allclose(E.rms_norm_heads(v, g, 0.0)[0, 0], -g, rtol=1e-15)
    assert np.allclose(E.rms_norm_heads(v, g, 9.0)[0, 0], -g / np.sqrt(2.0), rtol=1e-15)
    # a zero head stays zero for any eps > 0
    assert np.array_equal(E.rms_norm_heads(np.zeros((1, 1, D)), g, 1e-6), np.zeros((1, 1, D)))


def test_rotation_is_complex_multiplication():
    rng = np.random.default_rng(3)
    z = heads(rng, 6, 2)
    th, c, s = angles(rng, 6)
    got = E.rotate_pairs(z, c, s)
    zc = z[..., 0::2] + 1j * z[..., 1::2]
    want = zc * np.exp(1j * th)[:, None, :]
    assert np.allclose(got[..., 0::2], want.real, rtol=0, atol=1e-13)
    assert np.allclose(got[..., 1::2], want.imag, rtol=0, atol=1e-13)


def test_rotation_special_angles_and_composition():
    rng = np.random.default_rng(4)
    z = heads(rng, 3, 1)
    one, zero = np.ones((3, D // 2)), np.zeros((3, D // 2))
    assert np.array_equal(E.rotate_pairs(z, one, zero), z)
    q = E.rotate_pairs(z, zero, one)  # a quarter turn: (a, b) -> (-b, a)
    assert np.array_equal(q[..., 0::2], -z[..., 1::2]) and np.array_equal(q[..., 1::2], z[..., 0::2])
    # the unit pair (1, 0) goes to (cos, sin): the turn is counterclockwise
    e = np.zeros((3, 1, D))
    e[..., 0] = 1.0
    th, c, s = angles(rng, 3)
    r = E.rotate_pairs(e, c, s)
    assert np.array_equal(r[:, 0, 0], c[:, 0]) and np.array_equal(r[:, 0, 1], s[:, 0])
    # two turns add their angles, and every pair keeps its length
    th2 = rng.uniform(-np.pi, np.pi, (3, D // 2))
    twice = E.rotate_pairs(E.rotate_pairs(z, c, s), np.cos(th2), np.sin(th2))
    once = E.rotate_pairs(z, np.cos(th + th2), np.sin(th + th2))
    assert np.allclose(twice, once, rtol=0, atol=1e-13)
    lengths = lambda a: a[..., 0::2] ** 2 + a[..., 1::2] ** 2
    assert np.allclose(lengths(E.rotate_pairs(z, c, s)), lengths(z), rtol=1e-13)


def test_layout_of_q_k_v():
    """Q's heads get norm_q, K's norm_k, V is untouched; heads are contiguous
    blocks of 128 columns in the order Q, K, V."""
    rng = np.random.default_rng(5)
    M, H = 4, 3
    y = rng.standard_normal((M, 3 * H * D)) * 4.0
    gq, gk = rng.uniform(0.5, 2.0, D), rng.uniform(0.5, 2.0, D)
    th, c, s = angles(rng, M)
    out = E.qkv_norm_rope(y, H, gq, gk, 1e-6, c, s)
    assert np.array_equal(out[:, 2 * H * D:], y[:, 2 * H * D:])
    for part, g in ((0, gq), (1, gk)):
        for h in range(H):
            cols = slice((part * H + h) * D, (part * H + h + 1) * D)
            v = y[:, cols]
            z = v / np.sqrt(np.mean(v * v, axis=1, keepdims=True) + 1e-6) * g
            zc = (z[:, 0::2] + 1j * z[:, 1::2]) * np.exp(1j * th)
            assert np.allclose(out[:, cols][:, 0::2], zc.real, rtol=0, atol=1e-12)
            assert np.allclose(out[:, cols][:, 1::2], zc.imag, rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        E.qkv_norm_rope(y[:, :-D], H, gq, gk, 1e-6, c, s)


def test_norm_comes_before_the_rotation():
    """With a non-uniform gamma the order matters; the attention code normalizes
    first. Rotating first and normalizing after gives a different result."""
    rng = np.random.default_rng(6)
    y = rng.standard_normal((2, 3 * D))
    g = rng.uniform(0.2, 3.0, D)
    th, c, s = angles(rng, 2)
    out = E.qkv_norm_rope(y, 1, g, g, 0.0, c, s)
    other = E.rms_norm_heads(E.rotate_pairs(y[:, :D].reshape(2, 1, D), c, s), g, 0.0).reshape(2, D)
    assert not np.allclose(out[:, :D], other, atol=1e-6)
