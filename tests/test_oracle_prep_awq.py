"""Pins for the oracle's offline prep and AWQ: defining properties of the
smoothing factor and the SVD split, and closed forms / brute force for AWQ."""

import numpy as np

import workloads as WL
from oracle import awq as A
from oracle import formats as F
from oracle import prep as P


def _small_layer(seed=0):
    shape = WL.custom_svdq("t", 96, 128, 80, 16, seed=seed, n_outliers=3,
                           outlier_scale=30.0, spike_rank=4, spike_sv=5.0)
    return WL.svdq_inputs(shape)


def test_smoothing_balances_channel_maxima():
    d = _small_layer()
    x, w = F.bf16_from_bits(d["X"]), F.bf16_from_bits(d["W"])
    lam, si = P.smoothing_factors(x, w)
    xmax = np.abs(x).max(0) / lam
    wmax = np.abs(w).max(0) * lam
    assert np.allclose(xmax, wmax, rtol=1e-12)       # the defining property of alpha = 0.5
    assert np.allclose(si, 1 / lam, rtol=2 ** -24)
    # a dead channel keeps lambda = 1
    x[:, 5] = 0.0
    lam2, _ = P.smoothing_factors(x, w)
    assert lam2[5] == 1.0


def test_smoothing_preserves_the_product():
    d = _small_layer(1)
    out = P.prepare_svdq_layer("nvfp4", d["X"], d["W"], 16)
    x, w = F.bf16_from_bits(d["X"]), F.bf16_from_bits(d["W"])
    from oracle.svdq import smooth
    xh = smooth(x, out["smooth_inv"])
    ref = x @ w.T
    assert np.abs(xh @ out["w_hat"].T - ref).max() <= 1e-6 * np.abs(ref).max()


def test_svd_split_is_best_rank_r():
    d = _small_layer(2)
    out = P.prepare_svdq_layer("nvfp4", d["X"], d["W"], 16)
    wh = out["w_hat"]
    s = np.linalg.svd(wh, compute_uv=False)
    tail = np.sqrt(np.sum(s[16:] ** 2))
    resid = np.linalg.norm(wh - (out["L1"] @ out["L2"]).T)
    # Eckart-Young up to the bf16 rounding of the two factors
    assert abs(resid - tail) <= 6 * 2 ** -9 * np.sqrt(np.sum(s[:16] ** 2))
    assert resid < np.linalg.norm(wh)
    # rank 0 leaves the whole matrix as residual
    out0 = P.prepare_svdq_layer("nvfp4", d["X"], d["W"], 0)
    assert np.array_equal(out0["R"], F.bf16_round(out0["w_hat"]))


def test_awq_quantize_properties():
    rng = np.random.default_rng(3)
    w = F.bf16_round(rng.standard_normal((24, 256)) * 0.02)
    q, s, z = A.quantize_weight(w)
    assert q.min() >= 0 and q.max() <= 15
    assert np.array_equal(F.bf16_round(s), s) and np.all(z == np.rint(z))
    assert not np.any(np.signbit(z))  # integer zero points: a zero is +0
    # a constant positive group: s = 1, rint(-min) = -0 becomes the integer +0
    qc, sc, zc = A.quantize_weight(np.full((1, 64), 0.125))
    assert sc[0, 0] == 1.0 and zc[0, 0] == 0.0 and not np.signbit(zc[0, 0]) and not qc.any()
    deq = A.dequant_weight(q, s, z)
    # codes strictly inside (0, 15) come from rint: error at most half a step
    sv = np.repeat(s, 64, axis=1)
    inner = (q > 0) & (q < 15)
    assert np.all(np.abs(deq - w)[inner] <= 0.5 * sv[inner] * (1 + 1e-12))
    # in groups that straddle zero the clamp can only add the bf16 rounding of
    # s over the 15-step range: at most 15 s 2^-8 more
    g = w.reshape(24, 4, 64)
    straddle = np.repeat((g.min(2) <= 0) & (g.max(2) >= 0), 64, axis=1)
    assert np.all(np.abs(deq - w)[straddle] <= (0.5 + 15 * 2 ** -8) * sv[straddle])


def test_awq_closed_forms():
    K = 128
    q = np.full((3, K), 15, dtype=np.uint8)
    s = np.ones((3, 2))
    z = np.zeros((3, 2))
    x = np.ones((2, K))
    b = np.array([1.0, -2.0, 0.5])
    assert np.array_equal(A.linear(x, q, s, z, b), np.tile(15.0 * K + b, (2, 1)))
    # zero point equal to the code cancels it
    z8 = np.full((3, 2), 15.0)
    assert not A.linear(x, q, s, z8).any()
    # a constant group uses s = 1
    qc, sc, zc = A.quantize_weight(np.full((1, 64), -3.0))
    assert sc[0, 0] == 1.0 and zc[0, 0] == 3.0 and not qc.any()


def test_awq_brute_force_small():
    rng = np.random.default_rng(4)
    M, N, K = 2, 3, 128
    x = F.bf16_round(rng.standard_normal((M, K)))
    w = F.bf16_round(rng.standard_normal((N, K)) * 0.02)
    q, s, z = A.quantize_weight(w)
    b = F.bf16_round(rng.standard_normal(N) * 0.1)
    y = A.linear(x, q, s, z, b)
    for m in range(M):
        for n in range(N):
            acc = b[n]
            for k in range(K):
                acc += x[m, k] * (int(q[n, k]) - z[n, k // 64]) * s[n, k // 64]
            assert abs(acc - y[m, n]) <= 1e-12 * max(1, abs(acc))
