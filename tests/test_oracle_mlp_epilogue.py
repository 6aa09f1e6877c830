"""Pins of the oracle's fused MLP (fc1 -> GELU -> fc2's 4-bit input) against
facts that do not restate its formulas: torch's own GELU (both forms) as an
independent library routine, the identity GELU(y) - GELU(-y) = y, the known gap
between the tanh and erf forms, exact power-of-two smoothing, and the whole
quantized MLP against the unquantized float64 MLP it approximates (dropping
GELU, the bias or the smoothing direction would fail it)."""

import numpy as np
import pytest

from oracle import formats as F
from oracle import mlp_epilogue as ME
from oracle import prep as P
from oracle import svdq as S

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("form", ["tanh", "none"])
def test_gelu_matches_torch(form):
    y = np.concatenate([np.linspace(-12, 12, 4001), np.random.default_rng(0).standard_normal(1000) * 3])
    want = torch.nn.functional.gelu(torch.from_numpy(y), approximate=form).numpy()
    assert np.max(np.abs(ME.gelu(y, form) - want)) <= 4 * np.finfo(np.float64).eps * np.maximum(1, np.abs(y)).max()


@pytest.mark.parametrize("form", ["tanh", "none"])
def test_gelu_odd_part_is_the_identity(form):
    # Phi(y) + Phi(-y) = 1 for the exact form, and tanh is odd for the approximate one
    y = np.random.default_rng(1).standard_normal(500) * 4
    assert np.allclose(ME.gelu(y, form) - ME.gelu(-y, form), y, rtol=1e-15, atol=1e-15)
    assert ME.gelu(np.array([0.0]), form)[0] == 0.0


def test_tanh_form_is_the_approximation_not_erf():
    y = np.linspace(-8, 8, 160001)
    gap = np.max(np.abs(ME.gelu(y, "tanh") - ME.gelu(y, "none")))
    assert 4e-4 < gap < 5e-4  # the tanh form's known worst case, near |y| = 2.7
    with pytest.raises(ValueError):
        ME.gelu(y, "sigmoid")


def test_hidden_is_one_float32_rounding_then_smoothing():
    rng = np.random.default_rng(2)
    y1 = rng.standard_normal((6, 64)) * 3
    h = ME.hidden(y1, None)
    assert np.array_equal(h, h.astype(np.float32).astype(np.float64))
    assert np.all(np.abs(h - ME.gelu(y1)) <= np.abs(ME.gelu(y1)) * 2.0 ** -24)
    k = rng.integers(-5, 6, 64)
    assert np.array_equal(ME.hidden(y1, 2.0 ** k), h * 2.0 ** k[None, :])


def test_fc1_epilogue_outputs():
    rng = np.random.default_rng(3)
    y1 = rng.standard_normal((5, 128)) * 2
    si = F.rn32(rng.uniform(0.5, 2.0, 128))
    L1 = F.bf16_round(rng.standard_normal((128, 16)) * 0.1)
    ep = ME.fc1_epilogue(y1, si, L1)
    # the 4-bit codes decode to h_hat within NVFP4's error
    deq = S.dequant_nvfp4(ep["codes"], ep["scales"])
    assert np.linalg.norm(deq - ep["h_hat"]) < 0.15 * np.linalg.norm(ep["h_hat"])
    # xl1 against a brute-force loop
    want = np.array([[sum(ep["h_hat"][m, k] * L1[k, j] for k in range(128)) for j in range(16)]
                     for m in range(5)])
    assert np.allclose(ep["xl1"], want, rtol=1e-13, atol=1e-13)
    assert ME.fc1_epilogue(y1, si, np.zeros((128, 0)))["xl1"] is None


def test_fused_mlp_approximates_the_float64_mlp():
    """fc2 with smoothing from the hidden activation's channel maxima, an SVD
    split and a 4-bit residual, run on fc1's output through the fused
    epilogue, stays within the format's error of gelu(y1) W2^T + b2."""
    rng = np.random.default_rng(4)
    M, N1, N2, r = 64, 512, 256, 16
    y1 = rng.standard_normal((M, N1)) * 1.5
    y1[:, rng.permutation(N1)[:8]] *= 20.0  # outlier channels in the hidden activation
    w2 = F.bf16_round(rng.standard_normal((N2, N1)) * 0.02)
    b2 = F.bf16_round(rng.standard_normal(N2) * 0.5)
    h = ME.gelu(y1)
    _, si2 = P.smoothing_factors(h, w2)
    w2_hat = w2 * (1.0 / si2)[None, :]
    L1, L2 = P.svd_split(w2_hat, r)
    R = F.bf16_round(w2_hat - (L1 @ L2).T)
    qw, sw = S.quantize_nvfp4(R)
    got = ME.mlp_forward(y1, si2, L1, L2, qw, sw, b2)["Y"]
    want = h @ w2.T + b2[None, :]
    err = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err < 0.06
    # the same pipeline without GELU, without the bias or with the smoothing
    # inverted is far off
    no_gelu = S.w4a4_linear(S.dequant_nvfp4(*S.quantize_nvfp4(F.rn32(y1 * si2))),
                            S.dequant_nvfp4(qw, sw), F.rn32(y1 * si2) @ L1, L2, b2)
    assert np.linalg.norm(no_gelu - want) / np.linalg.norm(want) > 0.3
    no_bias = ME.mlp_forward(y1, si2, L1, L2, qw, sw, None)["Y"]
    assert np.linalg.norm(no_bias - want) / np.linalg.norm(want) > 5 * err
    flipped = ME.mlp_forward(y1, 1.0 / si2, L1, L2, qw, sw, b2)["Y"]
    assert np.linalg.norm(flipped - want) / np.linalg.norm(want) > 0.3
