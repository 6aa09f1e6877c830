"""The fused QKV epilogue (per-head RMS norm of Q and K, then the pairwise
rotation, in the NVFP4 GEMM's epilogue) through the C ABI:

* against the oracle's whole forward (layer, then the epilogue) on small
  layers that span several tiles and a ragged tail, with one or two CTAs per
  tile, an odd head count (a tile holding the last Q head and the first K
  head), bf16 and float32 output, with and without head weights and rotation;
* the V columns byte for byte equal to the plain linear's;
* at the full FLUX-like QKV size (M = 4608, K = 3072, N = 9216, r = 32) in the
  launch configuration the benchmark times: V byte for byte, and Q, K on
  sampled rows against the oracle's epilogue applied to the plain linear's
  float32 output.
"""

import numpy as np
import pytest

import workloads as WL
from oracle import formats as F
from oracle import layout as LO
from oracle import qkv_epilogue as E
from oracle import svdq as S
from tests import svdq_cases as C

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
D = E.HEAD_DIM


@pytest.fixture(scope="module")
def bq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_quantized_diffusion_b200 as bq
    return bq


def run_layer(bq, layer, ep, fused: bool, out_f32: bool, weights: bool, rope: bool):
    shape = layer["shape"]
    X = C.bf16_tensor(layer["x_bits"])
    si = C.f32_tensor(layer["smooth_inv"])
    L1s = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si) if shape.r else None
    codes, scales, xl1 = bq.svdq_quantize_act(X, L1s, si)
    wc = C.u8_tensor(C.tiled_codes("nvfp4", layer["w_codes"]))
    ws = C.u8_tensor(C.tiled_scales("nvfp4", layer["w_scales"]))
    L2 = C.bf16_tensor(F.bf16_bits(layer["L2"])) if shape.r else None
    bias = C.bf16_tensor(layer["bias_bits"])
    dt = torch.float32 if out_f32 else torch.bfloat16
    if not fused:
        return bq.svdq_w4a4_linear(codes, scales, xl1, wc, ws, L2, bias, M=shape.M, N_=shape.N,
                                   K=shape.K, out_dtype=dt)
    gq = C.bf16_tensor(ep["norm_q"]) if weights else None
    gk = C.bf16_tensor(ep["norm_k"]) if weights else None
    cos = angle_major(ep["cos"]) if rope else None
    sin = angle_major(ep["sin"]) if rope else None
    return bq.svdq_w4a4_linear_qkv_norm_rope(codes, scales, xl1, wc, ws, L2, bias, gq, gk, cos, sin,
                                             shape.M, shape.N, shape.K, eps=1e-6, out_dtype=dt)


def angle_major(table):
    """The oracle's [M, 64] angle table in the call's angle-major [64, M] layout."""
    return C.f32_tensor(np.ascontiguousarray(table.T))


def as_f64(y):
    return y.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M,H,K,r,out_f32,weights,rope", [
    (300, 2, 640, 32, False, True, True),     # ragged tail, CTA pairs, 3 column tiles
    (520, 3, 512, 16, True, True, True),      # odd head count: a tile holds Q's last and K's first head
    (256, 1, 512, 0, False, False, False),    # no low-rank branch, weight 1, no rotation
    (100, 2, 256, 32, False, True, True),     # M <= 128: one CTA per tile
    (1100, 4, 1024, 32, False, True, True),   # several row tiles, every CTA several tiles
])
def test_fused_qkv_matches_the_oracle(bq, M, H, K, r, out_f32, weights, rope):
    N = 3 * H * D
    shape = WL.custom_svdq(f"qkv_{M}_{H}", M, K, N, r, seed=60 + M, n_outliers=8,
                           outlier_scale=50.0, spike_rank=8, spike_sv=5.0)
    layer = C.oracle_layer(shape)
    ep = WL.qkv_epilogue_inputs(M, seed=70 + M)
    y = run_layer(bq, layer, ep, True, out_f32, weights, rope)
    assert bq.svdq_check_device_status() == 0
    fwd = S.svdq_forward("nvfp4", layer["x_bits"], layer["smooth_inv"], layer["L1"] if r else None,
                         layer["L2"] if r else None, layer["w_codes"], layer["w_scales"],
                         layer["bias_bits"])
    gq = F.bf16_from_bits(ep["norm_q"]) if weights else None
    gk = F.bf16_from_bits(ep["norm_k"]) if weights else None
    ref = E.qkv_norm_rope(fwd["Y"], H, gq, gk, 1e-6, ep["cos"] if rope else None,
                          ep["sin"] if rope else None)
    got = as_f64(y)
    qk = slice(0, 2 * H * D)
    C.assert_gemm_close(got[:, qk], ref[:, qk], bf16_out=not out_f32, what="Q, K")
    C.assert_gemm_close(got[:, 2 * H * D:], ref[:, 2 * H * D:], bf16_out=not out_f32, what="V")
    # V is the plain linear's output, byte for byte
    plain = run_layer(bq, layer, ep, False, out_f32, weights, rope)
    assert torch.equal(y[:, 2 * H * D:], plain[:, 2 * H * D:])


def test_unit_weights_give_unit_mean_square_heads(bq):
    """Weight 1, eps 0 and any rotation: every Q and K head of every row has mean
    square 1 (rotation keeps each pair's length), up to float32 rounding."""
    M, H, K = 260, 2, 512
    shape = WL.custom_svdq("qkv_unit", M, K, 3 * H * D, 16, seed=81)
    layer = C.oracle_layer(shape)
    ep = WL.qkv_epilogue_inputs(M, seed=82)
    X = C.bf16_tensor(layer["x_bits"])
    si = C.f32_tensor(layer["smooth_inv"])
    L1s = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si)
    codes, scales, xl1 = bq.svdq_quantize_act(X, L1s, si)
    y = bq.svdq_w4a4_linear_qkv_norm_rope(
        codes, scales, xl1, C.u8_tensor(C.tiled_codes("nvfp4", layer["w_codes"])),
        C.u8_tensor(C.tiled_scales("nvfp4", layer["w_scales"])),
        C.bf16_tensor(F.bf16_bits(layer["L2"])), C.bf16_tensor(layer["bias_bits"]), None, None,
        angle_major(ep["cos"]), angle_major(ep["sin"]), M, 3 * H * D, K, eps=0.0,
        out_dtype=torch.float32)
    assert bq.svdq_check_device_status() == 0
    heads = as_f64(y)[:, :2 * H * D].reshape(M, 2 * H, D)
    ms = np.mean(heads * heads, axis=-1)
    assert np.max(np.abs(ms - 1.0)) < 1e-5


@pytest.mark.slow
def test_full_size_flux_qkv(bq):
    """M = 4608, K = 3072, N = 9216 (24 heads each), r = 32: weights from the
    library's own prep, the bench's launch configuration; Q and K on six sampled
    128-row blocks against the oracle's layer followed by its epilogue."""
    from bit_quantized_diffusion_b200 import prep
    shape = WL.QKV
    M, K, N, r, H = shape.M, shape.K, shape.N, shape.r, shape.N // (3 * D)
    d = WL.svdq_inputs(shape)
    X = C.bf16_tensor(d["X"])
    W = C.bf16_tensor(d["W"])
    bias = C.bf16_tensor(d["bias"])
    w = prep.prepare_svdq_weights(W, bq.svdq_column_absmax(X), r, "nvfp4")
    codes, scales, xl1 = bq.svdq_quantize_act(X, w["L1s"], w["smooth_inv"])
    ep = WL.qkv_epilogue_inputs(M, seed=90, angles="positions")
    gq, gk = C.bf16_tensor(ep["norm_q"]), C.bf16_tensor(ep["norm_k"])
    cos, sin = angle_major(ep["cos"]), angle_major(ep["sin"])
    y = bq.svdq_w4a4_linear_qkv_norm_rope(codes, scales, xl1, w["w_codes"], w["w_scales"], w["L2"],
                                          bias, gq, gk, cos, sin, M, N, K)
    plain = bq.svdq_w4a4_linear(codes, scales, xl1, w["w_codes"], w["w_scales"], w["L2"], bias,
                                M=M, N_=N, K=K)
    plain32 = bq.svdq_w4a4_linear(codes, scales, xl1, w["w_codes"], w["w_scales"], w["L2"], bias,
                                  M=M, N_=N, K=K, out_dtype=torch.float32)
    assert bq.svdq_check_device_status() == 0
    assert torch.equal(y[:, 2 * H * D:], plain[:, 2 * H * D:])
    blocks = np.unique(np.linspace(0, M // 128 - 1, 6).round().astype(int))
    rows = np.unique(np.concatenate([np.arange(b * 128, b * 128 + 128) for b in blocks] + [[M - 1]]))
    # the oracle's layer on those rows, with the weights the library prepared (in the
    # oracle's plain formats), followed by the oracle's epilogue
    bits = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)  # noqa: E731
    w_codes = S.unpack_nibbles(w["w_codes"].cpu().numpy().reshape(N, K // 2))
    w_scales = LO.untile_nvfp4_scales(w["w_scales"].cpu().numpy(), N, K)
    fwd = S.svdq_forward("nvfp4", d["X"][rows], w["smooth_inv"].cpu().numpy().astype(np.float64),
                         F.bf16_from_bits(bits(w["L1"])), F.bf16_from_bits(bits(w["L2"])), w_codes, w_scales,
                         d["bias"])
    ref = E.qkv_norm_rope(fwd["Y"], H, F.bf16_from_bits(ep["norm_q"]), F.bf16_from_bits(ep["norm_k"]), 1e-6,
                          ep["cos"][rows], ep["sin"][rows])
    C.assert_gemm_close(as_f64(y[rows])[:, :2 * H * D], ref[:, :2 * H * D], bf16_out=True,
                        what="Q, K (full size)")
    # and the plain call's float32 output through the same epilogue (the epilogue alone)
    ref32 = E.qkv_norm_rope(as_f64(plain32[rows]), H, F.bf16_from_bits(ep["norm_q"]),
                            F.bf16_from_bits(ep["norm_k"]), 1e-6, ep["cos"][rows], ep["sin"][rows])
    C.assert_gemm_close(as_f64(y[rows])[:, :2 * H * D], ref32[:, :2 * H * D], bf16_out=True,
                        what="Q, K against the plain call's epilogue")


def test_layer_class_matches_the_oracle(bq):
    """SvdqQkvNormRope on oracle-prepared weights (one call per forward after the
    quantizer), against the oracle's layer followed by its epilogue."""
    from bit_quantized_diffusion_b200.layers import SvdqQkvNormRope
    M, H, K, r = 384, 2, 1024, 32
    shape = WL.custom_svdq("qkv_layer", M, K, 3 * H * D, r, seed=91, n_outliers=8,
                           outlier_scale=50.0, spike_rank=8, spike_sv=5.0)
    layer = C.oracle_layer(shape)
    ep = WL.qkv_epilogue_inputs(M, seed=92)
    si = C.f32_tensor(layer["smooth_inv"])
    w = {"smooth_inv": si, "L1s": bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si),
         "L2": C.bf16_tensor(F.bf16_bits(layer["L2"])),
         "w_codes": C.u8_tensor(C.tiled_codes("nvfp4", layer["w_codes"])),
         "w_scales": C.u8_tensor(C.tiled_scales("nvfp4", layer["w_scales"])),
         "fmt": "nvfp4", "N": shape.N, "K": K, "r": r}
    mod = SvdqQkvNormRope(w, C.bf16_tensor(layer["bias_bits"]), max_tokens=512,
                          norm_q=C.bf16_tensor(ep["norm_q"]), norm_k=C.bf16_tensor(ep["norm_k"]))
    y = mod(C.bf16_tensor(layer["x_bits"]), angle_major(ep["cos"]), angle_major(ep["sin"]))
    assert bq.svdq_check_device_status() == 0
    fwd = S.svdq_forward("nvfp4", layer["x_bits"], layer["smooth_inv"], layer["L1"], layer["L2"],
                         layer["w_codes"], layer["w_scales"], layer["bias_bits"])
    ref = E.qkv_norm_rope(fwd["Y"], H, F.bf16_from_bits(ep["norm_q"]), F.bf16_from_bits(ep["norm_k"]),
                          1e-6, ep["cos"], ep["sin"])
    got = as_f64(y)
    C.assert_gemm_close(got[:, :2 * H * D], ref[:, :2 * H * D], bf16_out=True, what="Q, K (layer)")
    C.assert_gemm_close(got[:, 2 * H * D:], ref[:, 2 * H * D:], bf16_out=True, what="V (layer)")
