"""Offline weight preparation on the GPU (svdq_column_absmax, svdq_smoothing,
svdq_lowrank_factors, svdq_residual, awq_quantize_weight, and prep.py, which
strings them around the SVD) against the oracle's prep (oracle/prep.py,
oracle/awq.py): the smoothing vector, the bf16 factors, the residual and the
AWQ codes, scales and zero points bit for bit, from small ragged shapes with
zero channels and constant groups up to the weights the benchmark times."""

import numpy as np
import pytest

import workloads as WL
from oracle import awq as OA
from oracle import formats as F
from oracle import layout as LO
from oracle import prep as P
from oracle import svdq as S
from tests import svdq_cases as C

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_quantized_diffusion_b200 as bq
    return bq


def _f32(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("rows,K", [(1, 8), (37, 520), (1000, 1024)])
def test_column_absmax_is_exact(bq, rows, K):
    rng = np.random.default_rng(rows + K)
    a_bits = WL.to_bf16_bits(rng.standard_normal((rows, K)) * rng.uniform(0.1, 10.0, K))
    a_bits[:, 0] = 0x8000  # a column of negative zeros: max 0
    got = bq.svdq_column_absmax(C.bf16_tensor(a_bits))
    want = np.max(np.abs(F.bf16_from_bits(a_bits)), axis=0)
    assert np.array_equal(_f32(got), want)


def _layer(seed, M, N, K, zero_x_col=None, zero_w_col=None):
    sh = WL.custom_svdq("prep", M, K, N, 16, seed=seed, n_outliers=4, outlier_scale=30.0,
                        spike_rank=4, spike_sv=2.0)
    d = WL.svdq_inputs(sh)
    if zero_x_col is not None:
        d["X"][:, zero_x_col] = 0
    if zero_w_col is not None:
        d["W"][:, zero_w_col] = 0
    return d


def test_smoothing_matches_the_oracle(bq):
    d = _layer(5, 300, 272, 1024, zero_x_col=5, zero_w_col=7)
    x, w = F.bf16_from_bits(d["X"]), F.bf16_from_bits(d["W"])
    _, want = P.smoothing_factors(x, w)
    xa = bq.svdq_column_absmax(C.bf16_tensor(d["X"]))
    got = bq.svdq_smoothing(xa, C.bf16_tensor(d["W"]))
    g = _f32(got)
    assert g[5] == 1.0 and g[7] == 1.0  # a zero maximum leaves the channel unsmoothed
    assert np.array_equal(g, want)


@pytest.mark.parametrize("N,K,r", [(272, 1024, 32), (96, 320, 16), (200, 64, 48)])
def test_factors_and_residual_match_the_oracle(bq, N, K, r):
    d = _layer(10 + r, 128, N, K)
    x, w = F.bf16_from_bits(d["X"]), F.bf16_from_bits(d["W"])
    _, smooth_inv = P.smoothing_factors(x, w)
    w_hat = w * (1.0 / smooth_inv)[None, :]
    L1, L2 = P.svd_split(w_hat, r)
    # the same float64 SVD the oracle's split used, handed to the GPU
    u, s, vt = np.linalg.svd(w_hat, full_matrices=False)
    tt = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    gL1, gL2 = bq.svdq_lowrank_factors(tt(u), tt(s), tt(vt), r)
    assert np.array_equal(_f32(gL1), L1)
    assert np.array_equal(_f32(gL2), L2)
    si = C.f32_tensor(smooth_inv)
    R = bq.svdq_residual(C.bf16_tensor(d["W"]), si, C.bf16_tensor(F.bf16_bits(L1)),
                         C.bf16_tensor(F.bf16_bits(L2)))
    assert np.array_equal(_f32(R), P.residual(w_hat, L1, L2))
    R0 = bq.svdq_residual(C.bf16_tensor(d["W"]), si, None, None)  # rank 0: the smoothed weight
    assert np.array_equal(_f32(R0), F.bf16_round(w_hat))
    assert bq.svdq_check_device_status() == 0


def test_prepare_svdq_weights_against_the_oracle_prep(bq):
    """prep.prepare_svdq_weights (cuSOLVER's float64 SVD, the library for the rest)
    against the oracle's prep of the same layer: the smoothing vector bit for bit;
    the residual bit for bit given the GPU's own factors; the factors' product
    within bf16 rounding of the oracle's (singular vectors are unique up to sign,
    which the product does not see); the residual's codes and scales bit for bit
    against the oracle's quantizer."""
    from bit_quantized_diffusion_b200 import prep
    d = _layer(21, 512, 384, 1024)
    r = 32
    x, w = F.bf16_from_bits(d["X"]), F.bf16_from_bits(d["W"])
    ora = P.prepare_svdq_layer("nvfp4", d["X"], d["W"], r)
    X = C.bf16_tensor(d["X"])
    got = prep.prepare_svdq_weights(C.bf16_tensor(d["W"]), bq.svdq_column_absmax(X), r)
    assert np.array_equal(_f32(got["smooth_inv"]), ora["smooth_inv"])
    gL1, gL2 = _f32(got["L1"]), _f32(got["L2"])
    prod, prod_o = gL1 @ gL2, ora["L1"] @ ora["L2"]
    assert np.linalg.norm(prod - prod_o) / np.linalg.norm(prod_o) < 1e-2
    w_hat = w * (1.0 / ora["smooth_inv"])[None, :]
    R = _f32(got["R"])
    assert np.array_equal(R, P.residual(w_hat, gL1, gL2))
    q, sc = S.quantize("nvfp4", R)
    assert np.array_equal(got["w_codes"].cpu().numpy(), S.pack_nibbles(q).reshape(-1))
    assert np.array_equal(got["w_scales"].cpu().numpy(), LO.tile_nvfp4_scales(sc))
    assert bq.svdq_check_device_status() == 0


def _awq_check(bq, w_bits):
    q, s, z = OA.quantize_weight(F.bf16_from_bits(w_bits))
    N, K = w_bits.shape
    qt, szt = bq.awq_quantize_weight(C.bf16_tensor(w_bits))
    # the layouts svdq_pack(AWQ) writes, bit for bit
    assert np.array_equal(qt.cpu().numpy(), LO.tile_awq_qweight(q))
    assert np.array_equal(szt.cpu().numpy().view(np.uint16), LO.tile_awq_sz(F.bf16_bits(s), F.bf16_bits(z)))


def test_awq_quantizer_matches_the_oracle(bq):
    rng = np.random.default_rng(31)
    N, K = 100, 192
    w = rng.standard_normal((N, K)) * 0.02
    w[3, 0:64] = 0.125                      # a constant group: s = 1, z = 0
    w[4, 64:128] = -0.5                     # a constant negative group
    w[5, 128:192] = np.linspace(-1, 1, 64)  # exact endpoints
    w[6, :64] = np.abs(w[6, :64])           # all positive: z = 0
    w[7, :64] = -np.abs(w[7, :64])          # all negative: z = 15
    _awq_check(bq, WL.to_bf16_bits(w))


def test_awq_quantizer_at_the_adaln_width(bq):
    d = WL.awq_inputs(WL.AWQ_MOD)
    _awq_check(bq, d["W"])


@pytest.mark.slow
def test_prep_of_the_benchmarked_qkv_layer(bq):
    """The QKV layer's smoothing vector and residual (given the oracle's factors)
    as the benchmark prepares them, bit for bit against the oracle's prep."""
    layer = C.oracle_layer(WL.QKV)
    X = C.bf16_tensor(layer["x_bits"])
    W = C.bf16_tensor(layer["w_bits"])
    si = bq.svdq_smoothing(bq.svdq_column_absmax(X), W)
    assert np.array_equal(_f32(si), layer["smooth_inv"])
    R = bq.svdq_residual(W, si, C.bf16_tensor(F.bf16_bits(layer["L1"])),
                         C.bf16_tensor(F.bf16_bits(layer["L2"])))
    assert np.array_equal(_f32(R), layer["R"])
