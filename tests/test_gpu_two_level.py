"""Two-level NVFP4 through the C ABI against the oracle: the per-tensor scale
pair bit-exact, two-level codes and group scales bit-exact, the unit scale pair
reproducing the one-level calls byte for byte, and a layer whose activations
and residual weights lie far outside what E4M3 group scales alone can cover
(where the one-level format saturates and underflows) within the stated
tolerance of the oracle's two-level layer."""

import numpy as np
import pytest

import workloads as WL
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


def bf16_bits(a):
    return WL.to_bf16_bits(a)


@pytest.mark.parametrize("magnitude", [1.0, 3e5, 2e-9, 0.0])
@pytest.mark.parametrize("smoothed", [False, True])
def test_tensor_scale_matches_the_oracle(bq, magnitude, smoothed):
    rng = np.random.default_rng(7)
    M, K = 300, 640
    xb = bf16_bits(rng.standard_normal((M, K)) * magnitude)
    si = F.rn32(rng.uniform(0.5, 2.0, K)) if smoothed else None
    scale = bq.svdq_tensor_scale(C.bf16_tensor(xb), C.f32_tensor(si) if smoothed else None)
    assert bq.svdq_check_device_status() == 0
    got = scale.cpu().numpy().astype(np.float64)
    want = S.tensor_scale(S.smooth(F.bf16_from_bits(xb), si))
    assert (got[0], got[1]) == want


@pytest.mark.parametrize("magnitude", [1.0, 3e5, 2e-9])
def test_two_level_codes_and_scales_bit_exact(bq, magnitude):
    rng = np.random.default_rng(8)
    M, K = 300, 640
    xb = bf16_bits(rng.standard_normal((M, K)) * magnitude)
    si = F.rn32(rng.uniform(0.5, 2.0, K))
    X, sit = C.bf16_tensor(xb), C.f32_tensor(si)
    scale = bq.svdq_tensor_scale(X, sit)
    codes, scales, _ = bq.svdq_quantize_act_two_level(X, scale, None, sit)
    assert bq.svdq_check_device_status() == 0
    xhat = S.smooth(F.bf16_from_bits(xb), si)
    s_t, inv = S.tensor_scale(xhat)
    q, sc = S.quantize_nvfp4_two_level(xhat, inv)
    assert np.array_equal(codes.cpu().numpy(), S.pack_nibbles(q).reshape(-1))
    assert np.array_equal(scales.cpu().numpy(), LO.tile_nvfp4_scales(sc))


def test_unit_scale_pair_is_the_one_level_call(bq):
    shape = WL.custom_svdq("two_level_unit", 300, 640, 272, 32, seed=31)
    layer = C.oracle_layer(shape)
    X = C.bf16_tensor(layer["x_bits"])
    si = C.f32_tensor(layer["smooth_inv"])
    L1s = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si)
    one = torch.ones(2, dtype=torch.float32, device="cuda")
    c1, s1, x1 = bq.svdq_quantize_act(X, L1s, si)
    c2, s2, x2 = bq.svdq_quantize_act_two_level(X, one, L1s, si)
    assert torch.equal(c1, c2) and torch.equal(s1, s2) and torch.equal(x1, x2)
    wc, ws, _ = bq.svdq_quantize_act(C.bf16_tensor(F.bf16_bits(layer["R"])), None, None)
    L2 = C.bf16_tensor(F.bf16_bits(layer["L2"]))
    bias = C.bf16_tensor(layer["bias_bits"])
    y1 = bq.svdq_w4a4_linear(c1, s1, x1, wc, ws, L2, bias, M=shape.M, N_=shape.N, K=shape.K)
    y2 = bq.svdq_w4a4_linear_two_level(c2, s2, one, x2, wc, ws, one, L2, bias, shape.M, shape.N, shape.K)
    assert bq.svdq_check_device_status() == 0
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("M,N,K,r,out_f32", [(300, 272, 640, 32, False), (520, 384, 1024, 16, True),
                                             (2048, 2816, 512, 32, False)])
def test_out_of_range_layer_matches_the_oracle(bq, M, N, K, r, out_f32):
    """Activations around 1e5 (E4M3 group scales saturate) and weights around 1e-8
    (they underflow): the two-level layer stays within the stated tolerance."""
    rng = np.random.default_rng(40 + M)
    xb = bf16_bits(rng.standard_normal((M, K)) * 1.3e5)
    wb = bf16_bits(rng.standard_normal((N, K)) * 2e-8)
    bias_b = bf16_bits(rng.standard_normal(N) * 0.1)
    x, w = F.bf16_from_bits(xb), F.bf16_from_bits(wb)
    L1, L2 = P.svd_split(w, r)
    R = F.bf16_round(w - (L1 @ L2).T)
    # the oracle's layer: no smoothing, the tensor scales of x and R
    sa, inva = S.tensor_scale(x)
    sw, invw = S.tensor_scale(R)
    qa, sca = S.quantize_nvfp4_two_level(x, inva)
    qw, scw = S.quantize_nvfp4_two_level(R, invw)
    ref = S.w4a4_linear_two_level(S.dequant_nvfp4(qa, sca), S.dequant_nvfp4(qw, scw), sa, sw,
                                  S.down_proj(x, L1), L2, F.bf16_from_bits(bias_b))
    # the same layer through the library
    X = C.bf16_tensor(xb)
    Rt = C.bf16_tensor(F.bf16_bits(R))
    a_scale = bq.svdq_tensor_scale(X)
    w_scale = bq.svdq_tensor_scale(Rt)
    L1s = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(L1)), None)
    codes, scales, xl1 = bq.svdq_quantize_act_two_level(X, a_scale, L1s, None)
    wc, ws, _ = bq.svdq_quantize_act_two_level(Rt, w_scale)
    y = bq.svdq_w4a4_linear_two_level(codes, scales, a_scale, xl1, wc, ws, w_scale,
                                      C.bf16_tensor(F.bf16_bits(L2)), C.bf16_tensor(bias_b), M, N, K,
                                      out_dtype=torch.float32 if out_f32 else torch.bfloat16)
    assert bq.svdq_check_device_status() == 0
    assert np.array_equal(codes.cpu().numpy(), S.pack_nibbles(qa).reshape(-1))
    assert np.array_equal(wc.cpu().numpy(), S.pack_nibbles(qw).reshape(-1))
    assert np.array_equal(ws.cpu().numpy(), LO.tile_nvfp4_scales(scw))
    C.assert_gemm_close(y.float().cpu().numpy().astype(np.float64), ref, bf16_out=not out_f32,
                        what="two-level Y")
    # the one-level format cannot represent these tensors: its layer is far off
    q1, s1 = S.quantize_nvfp4(x)
    qw1, sw1 = S.quantize_nvfp4(R)
    one = S.w4a4_linear(S.dequant_nvfp4(q1, s1), S.dequant_nvfp4(qw1, sw1), S.down_proj(x, L1), L2,
                        F.bf16_from_bits(bias_b))
    assert C.rel_l2(one, ref) > 0.05


def test_layer_class_two_level_matches_the_oracle(bq):
    """SvdqW4A4Linear in two-level mode (per-call activation scale) on weights
    quantized two-level by the library, against the oracle's two-level layer."""
    from bit_quantized_diffusion_b200.layers import SvdqW4A4Linear
    shape = WL.custom_svdq("two_level_layer", 384, 1024, 512, 32, seed=33, n_outliers=8,
                           outlier_scale=50.0, spike_rank=8, spike_sv=5.0)
    layer = C.oracle_layer(shape)
    si = C.f32_tensor(layer["smooth_inv"])
    Rt = C.bf16_tensor(F.bf16_bits(layer["R"]))
    w_tscale = bq.svdq_tensor_scale(Rt)
    wc, ws, _ = bq.svdq_quantize_act_two_level(Rt, w_tscale)
    weights = {"smooth_inv": si, "L1s": bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si),
               "L2": C.bf16_tensor(F.bf16_bits(layer["L2"])), "w_codes": wc, "w_scales": ws,
               "w_tscale": w_tscale, "fmt": "nvfp4", "N": shape.N, "K": shape.K, "r": shape.r}
    lin = SvdqW4A4Linear(weights, C.bf16_tensor(layer["bias_bits"]), max_tokens=512)
    y = lin(C.bf16_tensor(layer["x_bits"]))
    assert bq.svdq_check_device_status() == 0
    xhat = S.smooth(F.bf16_from_bits(layer["x_bits"]), layer["smooth_inv"])
    sa, inva = S.tensor_scale(xhat)
    sw, invw = S.tensor_scale(layer["R"])
    qa, sca = S.quantize_nvfp4_two_level(xhat, inva)
    qw, scw = S.quantize_nvfp4_two_level(layer["R"], invw)
    ref = S.w4a4_linear_two_level(S.dequant_nvfp4(qa, sca), S.dequant_nvfp4(qw, scw), sa, sw,
                                  S.down_proj(xhat, layer["L1"]), layer["L2"],
                                  F.bf16_from_bits(layer["bias_bits"]))
    C.assert_gemm_close(y.float().cpu().numpy().astype(np.float64), ref, bf16_out=True,
                        what="two-level layer Y")


def test_prep_two_level_weights(bq):
    """prepare_svdq_weights(two_level=True): the residual's scale pair, codes and group
    scales bit-exact against the oracle on the residual prep returns, and the layer it
    makes (per-call activation scale) close to the unquantized product on weights too
    small for E4M3 group scales alone."""
    from bit_quantized_diffusion_b200 import prep
    from bit_quantized_diffusion_b200.layers import SvdqW4A4Linear
    rng = np.random.default_rng(51)
    M, N, K, r = 256, 384, 512, 32
    x = C.bf16_tensor(bf16_bits(rng.standard_normal((M, K)) * 3.0))
    w = C.bf16_tensor(bf16_bits(rng.standard_normal((N, K)) * 1e-7))
    wt = prep.prepare_svdq_weights(w, x.float().abs().amax(dim=0), r, "nvfp4", two_level=True)
    R = C.bf16_bits_of(wt["R"])
    Rd = F.bf16_from_bits(R)
    s_w, inv_w = S.tensor_scale(Rd)
    got = wt["w_tscale"].cpu().numpy().astype(np.float64)
    assert (got[0], got[1]) == (s_w, inv_w)
    q, sc = S.quantize_nvfp4_two_level(Rd, inv_w)
    assert np.array_equal(wt["w_codes"].cpu().numpy(), S.pack_nibbles(q).reshape(-1))
    assert np.array_equal(wt["w_scales"].cpu().numpy(), LO.tile_nvfp4_scales(sc))
    y = SvdqW4A4Linear(wt, None, max_tokens=M)(x)
    assert bq.svdq_check_device_status() == 0
    want = x.double() @ w.double().T
    assert float((y.double() - want).norm() / want.norm()) < 0.15
    with pytest.raises(ValueError):
        prep.prepare_svdq_weights(w, x.float().abs().amax(dim=0), r, "int4", two_level=True)
