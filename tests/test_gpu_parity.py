"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Codes and scales must be bit-exact. GEMM outputs: rel-L2 <= 2e-3 against the
unrounded oracle and max |err| <= 1e-2 rms(Y) (for bf16 output plus the output's
own rounding: 2^-9 on rel-L2, half a bf16 ulp on max-abs); the float32 output
mode must additionally agree to 1e-5 rel-L2,
since the 4-bit products are exact and only float32 accumulation and the
hi/lo low-rank split round.
"""

import numpy as np
import pytest

import workloads as WL
from oracle import awq as OA
from oracle import formats as F
from oracle import layout as LO
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


SMALL = [
    WL.custom_svdq("ragged", 300, 640, 272, 32, seed=11),
    WL.custom_svdq("tiny_r16", 256, 512, 512, 16, seed=12),
    WL.custom_svdq("one_row", 1, 128, 48, 16, seed=13),
    WL.custom_svdq("r0", 130, 256, 160, 0, seed=14),
    WL.custom_svdq("r256", 200, 512, 256, 256, seed=15, spike_rank=8, spike_sv=5.0),
    # more tiles than SMs: every persistent CTA walks several tiles, both accumulators
    WL.custom_svdq("many_tiles", 2048, 512, 2816, 32, seed=18),
    WL.custom_svdq("many_tiles_r128", 2176, 256, 2560, 128, seed=19),
    # K >= 8192 selects CTA-pair tiles (256 rows); M and N ragged in both halves
    WL.custom_svdq("long_k_pair", 400, 8192, 528, 32, seed=20),
]

SMALL_INT4 = [
    WL.custom_svdq("int4_ragged", 300, 640, 272, 32, fmt="int4", seed=16),
    # an odd number of 64-wide groups (the last stage holds one) and r % 32 == 16
    WL.custom_svdq("int4_odd_groups", 200, 576, 400, 16, fmt="int4", seed=24),
    WL.custom_svdq("int4_one_row", 1, 128, 48, 16, fmt="int4", seed=25),
    WL.custom_svdq("int4_r0", 130, 256, 160, 0, fmt="int4", seed=26),
    WL.custom_svdq("int4_r256", 200, 512, 256, 256, fmt="int4", seed=27, spike_rank=8, spike_sv=5.0),
    WL.custom_svdq("int4_many_tiles_r128", 2176, 256, 2560, 128, fmt="int4", seed=28),
    # at most 128 rows with more than 128 columns per tile: the CTA pair's second CTA holds
    # only rows past M, and the tile's second 128 weight rows must still be converted
    WL.custom_svdq("int4_few_rows_wide", 100, 640, 400, 32, fmt="int4", seed=29),
    WL.custom_svdq("int4_one_row_wide", 1, 256, 272, 16, fmt="int4", seed=30),
    WL.custom_svdq("int4_128_rows", 128, 512, 528, 48, fmt="int4", seed=31),
]


def _quantize_gpu(bq, layer, X_bits, fmt, with_lowrank=True, smooth=True):
    X = C.bf16_tensor(X_bits)
    si = C.f32_tensor(layer["smooth_inv"]) if smooth else None
    r = layer["L1"].shape[1] if with_lowrank else 0
    L1s = C.bf16_tensor(F.bf16_bits(LO.lowrank_operand(layer["L1"], layer["smooth_inv"] if smooth else None))) if r else None
    codes, scales, xl1 = bq.svdq_quantize_act(X, L1s, si, fmt=fmt)
    assert bq.svdq_check_device_status() == 0
    return codes.cpu().numpy(), scales.cpu().numpy(), (
        xl1.cpu().numpy().astype(np.float64) if xl1 is not None else None)


@pytest.mark.parametrize("shape", SMALL + SMALL_INT4[:2], ids=lambda s: s.name)
def test_quantize_act_matches_oracle(bq, shape):
    layer = C.oracle_layer(shape)
    x = F.bf16_from_bits(layer["x_bits"])
    xhat = S.smooth(x, layer["smooth_inv"])
    q, s = S.quantize(shape.fmt, xhat)
    codes, scales, xl1 = _quantize_gpu(bq, layer, layer["x_bits"], shape.fmt, shape.r > 0)
    want_codes = C.tiled_codes(shape.fmt, q)
    bad = np.nonzero(codes != want_codes)[0]
    assert bad.size == 0, f"{bad.size} code bytes differ, first at {bad[:5]}: {codes[bad[:5]]} vs {want_codes[bad[:5]]}"
    want_scales = C.tiled_scales(shape.fmt, s)
    bad = np.nonzero(scales != want_scales)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:5]}"
    if shape.r:
        ref = S.down_proj(xhat, layer["L1"])
        err = np.abs(xl1 - ref)
        assert np.all(err <= C.xl1_bound(xhat, layer["L1"])), f"xl1 max err {err.max():.3e}"


def test_weight_quantizer_mode(bq):
    """No smoothing, rank 0: the residual-weight quantizer."""
    shape = WL.custom_svdq("w", 272, 640, 64, 16, seed=17)
    layer = C.oracle_layer(shape)
    R_bits = F.bf16_bits(layer["R"])
    for fmt in ("nvfp4", "int4"):
        codes, scales, _ = _quantize_gpu(bq, layer, R_bits, fmt, with_lowrank=False, smooth=False)
        q, s = S.quantize(fmt, layer["R"])
        assert np.array_equal(codes, C.tiled_codes(fmt, q)), fmt
        assert np.array_equal(scales, C.tiled_scales(fmt, s)), fmt


def test_negative_values_rounding_to_zero_keep_sign(bq):
    """E2M1 conversion keeps the sign of a negative value that rounds to 0."""
    x = np.zeros((1, 64))
    x[0, 0] = 6.0
    x[0, 1:5] = [-0.1, -0.2, 0.1, -0.0]
    bits = F.bf16_bits(F.bf16_round(x))
    import torch as T
    codes, _, _ = bq.svdq_quantize_act(C.bf16_tensor(bits), None, None, fmt="nvfp4")
    q, _ = S.quantize_nvfp4(F.bf16_from_bits(bits))
    assert np.array_equal(codes.cpu().numpy(), S.pack_nibbles(q).reshape(-1))


def _gemm_inputs(layer, fmt):
    x = F.bf16_from_bits(layer["x_bits"])
    xhat = S.smooth(x, layer["smooth_inv"])
    qa, sa = S.quantize(fmt, xhat)
    r = layer["L1"].shape[1]
    xl1 = F.rn32(S.down_proj(xhat, layer["L1"])) if r else None
    return xhat, qa, sa, xl1


@pytest.mark.parametrize("shape", SMALL + SMALL_INT4, ids=lambda s: s.name)
@pytest.mark.parametrize("with_bias", [True, False])
def test_w4a4_linear_matches_oracle(bq, shape, with_bias):
    layer = C.oracle_layer(shape)
    fmt = shape.fmt
    xhat, qa, sa, xl1 = _gemm_inputs(layer, fmt)
    M, K = qa.shape
    Nn = layer["w_codes"].shape[0]
    r = layer["L1"].shape[1]
    bias = F.bf16_from_bits(layer["bias_bits"]) if with_bias else None
    ref = S.w4a4_linear(S.dequant(fmt, qa, sa), S.dequant(fmt, layer["w_codes"], layer["w_scales"]),
                        xl1, layer["L2"] if r else None, bias)
    args = dict(
        a_codes=C.u8_tensor(C.tiled_codes(fmt, qa)),
        a_scales=C.u8_tensor(C.tiled_scales(fmt, sa)),
        xl1=C.f32_tensor(xl1) if r else None,
        w_codes=C.u8_tensor(C.tiled_codes(fmt, layer["w_codes"])),
        w_scales=C.u8_tensor(C.tiled_scales(fmt, layer["w_scales"])),
        L2=C.bf16_tensor(F.bf16_bits(layer["L2"])) if r else None,
        bias=C.bf16_tensor(layer["bias_bits"]) if with_bias else None,
    )
    y32 = bq.svdq_w4a4_linear(**args, M=M, N_=Nn, K=K, fmt=fmt, out_dtype=torch.float32)
    y16 = bq.svdq_w4a4_linear(**args, M=M, N_=Nn, K=K, fmt=fmt, out_dtype=torch.bfloat16)
    assert bq.svdq_check_device_status() == 0
    y32 = y32.cpu().numpy().astype(np.float64)
    y16 = y16.float().cpu().numpy().astype(np.float64)
    # NVFP4 operands are exact on the tensor cores: only float32 accumulation
    # order separates the result from the oracle. INT4 operands are dequantized
    # to FP16 first, one rounding each (at most 2^-12 relative), so a product is
    # within 2^-11 relative; the bound is that, four times inside the stated
    # output tolerance (relative L2 <= 2e-3).
    bound = 1e-5 if fmt == "nvfp4" else 2.0 ** -11
    assert C.rel_l2(y32, ref) <= bound, f"float32 output rel-L2 {C.rel_l2(y32, ref):.3e}"
    C.assert_gemm_close(y32, ref, bf16_out=False, what="Y f32")
    C.assert_gemm_close(y16, ref, bf16_out=True, what="Y bf16")


def test_w4a4_exact_on_grid(bq):
    """Operands exactly on the NVFP4 grid with unit scales: every product and
    every partial sum is exact in float32, so the output must equal the oracle
    bit for bit. Any misplaced code, scale or tile shows up here."""
    rng = np.random.default_rng(21)
    M, Nn, K = 200, 272, 512
    qa = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    qw = rng.integers(0, 16, size=(Nn, K)).astype(np.uint8)
    # scales: 2^e with e in {-2..2}, varying per group so scale placement matters
    sa = F.ue4m3_encode(2.0 ** rng.integers(-2, 3, size=(M, K // 16)))
    sw = F.ue4m3_encode(2.0 ** rng.integers(-2, 3, size=(Nn, K // 16)))
    ref = S.w4a4_linear(S.dequant_nvfp4(qa, sa), S.dequant_nvfp4(qw, sw), None, None, None)
    y = bq.svdq_w4a4_linear(C.u8_tensor(S.pack_nibbles(qa).reshape(-1)),
                            C.u8_tensor(LO.tile_nvfp4_scales(sa)), None,
                            C.u8_tensor(S.pack_nibbles(qw).reshape(-1)),
                            C.u8_tensor(LO.tile_nvfp4_scales(sw)), None, None,
                            M=M, N_=Nn, K=K, out_dtype=torch.float32)
    y = y.cpu().numpy().astype(np.float64)
    bad = np.argwhere(y != ref)
    assert bad.size == 0, f"{len(bad)} outputs differ; first {bad[:4].tolist()}: {y[tuple(bad[0])]} vs {ref[tuple(bad[0])]}"


def test_w4a4_int4_exact_on_grid(bq):
    """INT4 operands with power-of-two FP16 scales: every group's partial sum is
    an exact integer, every scaled term and the float32 sum of the eight groups
    fit in 24 bits, so the output must equal the oracle bit for bit. This pins
    the code conversion, its K order, the scale placement and the exactness of
    the tensor-core partial products."""
    rng = np.random.default_rng(29)
    M, Nn, K = 200, 272, 512
    qa = rng.integers(-7, 8, size=(M, K))
    qw = rng.integers(-7, 8, size=(Nn, K))
    sa = 2.0 ** rng.integers(-2, 3, size=(M, K // 64))
    sw = 2.0 ** rng.integers(-2, 3, size=(Nn, K // 64))
    ref = S.w4a4_linear(S.dequant("int4", qa, sa), S.dequant("int4", qw, sw), None, None, None)
    y = bq.svdq_w4a4_linear(C.u8_tensor(C.tiled_codes("int4", qa)),
                            C.u8_tensor(C.tiled_scales("int4", sa)), None,
                            C.u8_tensor(C.tiled_codes("int4", qw)),
                            C.u8_tensor(C.tiled_scales("int4", sw)), None, None,
                            M=M, N_=Nn, K=K, fmt="int4", out_dtype=torch.float32)
    assert bq.svdq_check_device_status() == 0
    y = y.cpu().numpy().astype(np.float64)
    bad = np.argwhere(y != ref)
    assert bad.size == 0, f"{len(bad)} outputs differ; first {bad[:4].tolist()}: {y[tuple(bad[0])]} vs {ref[tuple(bad[0])]}"


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_end_to_end_layer(bq, fmt):
    """quantize_act then w4a4_linear, against the oracle's whole forward."""
    shape = WL.custom_svdq("e2e", 384, 1024, 512, 32, fmt=fmt, seed=22, n_outliers=8,
                           outlier_scale=50.0, spike_rank=8, spike_sv=5.0)
    layer = C.oracle_layer(shape)
    fwd = S.svdq_forward(fmt, layer["x_bits"], layer["smooth_inv"], layer["L1"], layer["L2"],
                         layer["w_codes"], layer["w_scales"], layer["bias_bits"])
    X = C.bf16_tensor(layer["x_bits"])
    si = C.f32_tensor(layer["smooth_inv"])
    L1s = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si)
    codes, scales, xl1 = bq.svdq_quantize_act(X, L1s, si, fmt=fmt)
    y = bq.svdq_w4a4_linear(codes, scales, xl1, C.u8_tensor(C.tiled_codes(fmt, layer["w_codes"])),
                            C.u8_tensor(C.tiled_scales(fmt, layer["w_scales"])),
                            C.bf16_tensor(F.bf16_bits(layer["L2"])), C.bf16_tensor(layer["bias_bits"]),
                            M=shape.M, N_=shape.N, K=shape.K, fmt=fmt)
    assert bq.svdq_check_device_status() == 0
    C.assert_gemm_close(y.float().cpu().numpy().astype(np.float64), fwd["Y"], bf16_out=True)


@pytest.mark.parametrize("r,with_smooth", [(16, True), (32, True), (128, False), (256, True)])
def test_pack_lowrank_matches_oracle(bq, r, with_smooth):
    rng = np.random.default_rng(40 + r)
    K = 320
    L1 = F.bf16_round(rng.standard_normal((K, r)) * 0.3)
    si = F.rn32(rng.uniform(0.05, 4.0, K)) if with_smooth else None
    got = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(L1)), C.f32_tensor(si) if with_smooth else None)
    want = F.bf16_bits(LO.lowrank_operand(L1, si))
    assert np.array_equal(C.bf16_bits_of(got), want)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_pack_unpack_round_trip(bq, fmt):
    rng = np.random.default_rng(23)
    rows, K = 200, 384
    if fmt == "nvfp4":
        codes = rng.integers(0, 256, size=rows * K // 2).astype(np.uint8)
        want_codes = codes
    else:
        q = rng.integers(-7, 8, size=(rows, K))
        codes = S.pack_nibbles(q).reshape(-1)          # plain: two's complement
        want_codes = C.tiled_codes("int4", q)          # tiled: the same bytes
    if fmt == "nvfp4":
        plain = rng.integers(0, 127, size=(rows, K // 16)).astype(np.uint8)
        want = LO.tile_nvfp4_scales(plain)
        plain_t = C.u8_tensor(plain.reshape(-1))
    else:
        plain = F.fp16_round(rng.uniform(0, 2, size=(rows, K // 64)))
        want = LO.tile_int4_scales(plain).view(np.uint8)
        plain_t = C.u8_tensor(plain.astype(np.float16).view(np.uint8).reshape(-1))
    tc, ts = bq.svdq_pack("weight", fmt, rows, K, C.u8_tensor(codes), plain_t)
    assert np.array_equal(tc.cpu().numpy(), want_codes)
    assert np.array_equal(ts.cpu().numpy(), want)
    pc = torch.empty_like(C.u8_tensor(codes))
    ps = torch.empty_like(plain_t)
    bq.svdq_unpack("weight", fmt, rows, K, tc, ts, pc, ps)
    assert np.array_equal(pc.cpu().numpy(), codes)
    assert np.array_equal(ps.cpu().numpy(), plain_t.cpu().numpy())


def test_awq_pack_round_trip(bq):
    rng = np.random.default_rng(24)
    Nn, K = 40, 192
    q = rng.integers(0, 16, size=(Nn, K)).astype(np.uint8)
    s = rng.integers(0, 65535, size=(Nn, K // 64)).astype(np.uint16)
    z = rng.integers(0, 65535, size=(Nn, K // 64)).astype(np.uint16)
    qt, szt = bq.svdq_pack("awq", "nvfp4", Nn, K, C.u8_tensor(S.pack_nibbles(q).reshape(-1)),
                           C.u8_tensor(s.view(np.uint8).reshape(-1)),
                           C.u8_tensor(z.view(np.uint8).reshape(-1)))
    assert np.array_equal(qt.cpu().numpy(), LO.tile_awq_qweight(q))
    assert np.array_equal(szt.cpu().numpy().view(np.uint16), LO.tile_awq_sz(s, z))
    pq = torch.empty(Nn * K // 2, dtype=torch.uint8, device="cuda")
    ps = torch.empty(Nn * K // 64 * 2, dtype=torch.uint8, device="cuda")
    pz = torch.empty_like(ps)
    bq.svdq_unpack("awq", "nvfp4", Nn, K, qt, szt, pq, ps, pz)
    assert np.array_equal(pq.cpu().numpy(), S.pack_nibbles(q).reshape(-1))
    assert np.array_equal(ps.cpu().numpy().view(np.uint16).reshape(Nn, -1), s)
    assert np.array_equal(pz.cpu().numpy().view(np.uint16).reshape(Nn, -1), z)


def _awq_case(M, Nn, K, seed):
    rng = np.random.default_rng(seed)
    x_bits = WL.to_bf16_bits(rng.standard_normal((M, K)))
    w = F.bf16_round(rng.standard_normal((Nn, K)) * 0.02)
    q, s, z = OA.quantize_weight(w)
    b_bits = WL.to_bf16_bits(rng.standard_normal(Nn) * 0.1)
    return x_bits, q, s, z, b_bits


@pytest.mark.parametrize("M,Nn,K", [(4, 272, 640), (1, 64, 128), (8, 160, 192), (13, 96, 256),
                                    (64, 48, 128)])
def test_awq_matches_oracle(bq, M, Nn, K):
    x_bits, q, s, z, b_bits = _awq_case(M, Nn, K, 30 + M)
    ref = OA.linear(F.bf16_from_bits(x_bits), q, s, z, F.bf16_from_bits(b_bits))
    qt, szt = bq.svdq_pack("awq", "nvfp4", Nn, K, C.u8_tensor(S.pack_nibbles(q).reshape(-1)),
                           C.u8_tensor(F.bf16_bits(s).view(np.uint8).reshape(-1)),
                           C.u8_tensor(F.bf16_bits(z).view(np.uint8).reshape(-1)))
    y = bq.awq_w4a16_linear(C.bf16_tensor(x_bits), qt, szt, C.bf16_tensor(b_bits), Nn)
    assert bq.svdq_check_device_status() == 0
    C.assert_gemm_close(y.float().cpu().numpy().astype(np.float64), ref, bf16_out=True, what="AWQ Y")


def test_timeout_path_reports_and_recovers(bq):
    """A wait that nobody satisfies runs out (10 ms bound, nothing in flight);
    the status is reported once, then cleared, and the device keeps working."""
    assert bq.svdq_check_device_status() == 0
    bq.svdq_debug_wait_timeout(10000)
    assert bq.svdq_check_device_status() == 5
    assert bq.svdq_check_device_status() == 0
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    codes, scales, _ = bq.svdq_quantize_act(x, None, None)
    assert bq.svdq_check_device_status() == 0
    assert not codes.any() and not scales.any()


@pytest.mark.slow
def test_full_size_qkv_sampled(bq):
    """The FLUX-like QKV workload at full size, in the launch configuration the
    benchmark times: all codes and scales bit-exact, xl1 and Y on sampled rows."""
    shape = WL.QKV
    layer = C.oracle_layer(shape)
    x = F.bf16_from_bits(layer["x_bits"])
    X = C.bf16_tensor(layer["x_bits"])
    si = C.f32_tensor(layer["smooth_inv"])
    L1s = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si)
    wc, ws, _ = bq.svdq_quantize_act(C.bf16_tensor(F.bf16_bits(layer["R"])), None, None)
    codes, scales, xl1 = bq.svdq_quantize_act(X, L1s, si)
    y = bq.svdq_w4a4_linear(codes, scales, xl1, wc, ws, C.bf16_tensor(F.bf16_bits(layer["L2"])),
                            C.bf16_tensor(layer["bias_bits"]), M=shape.M, N_=shape.N, K=shape.K)
    assert bq.svdq_check_device_status() == 0
    assert np.array_equal(wc.cpu().numpy(), S.pack_nibbles(layer["w_codes"]).reshape(-1))
    assert np.array_equal(ws.cpu().numpy(), LO.tile_nvfp4_scales(layer["w_scales"]))
    xhat = S.smooth(x, layer["smooth_inv"])
    q, sc = S.quantize_nvfp4(xhat)
    assert np.array_equal(codes.cpu().numpy(), S.pack_nibbles(q).reshape(-1))
    assert np.array_equal(scales.cpu().numpy(), LO.tile_nvfp4_scales(sc))
    rows = np.unique(np.concatenate([np.arange(0, shape.M, 97), [shape.M - 1]]))
    ref_xl1 = S.down_proj(xhat[rows], layer["L1"])
    got_xl1 = xl1.cpu().numpy()[rows].astype(np.float64)
    assert np.all(np.abs(got_xl1 - ref_xl1) <= C.xl1_bound(xhat[rows], layer["L1"]))
    ref = S.w4a4_linear(S.dequant_nvfp4(q[rows], sc[rows]),
                        S.dequant_nvfp4(layer["w_codes"], layer["w_scales"]),
                        S.down_proj(xhat[rows], layer["L1"]), layer["L2"],
                        F.bf16_from_bits(layer["bias_bits"]))
    C.assert_gemm_close(y.float().cpu().numpy()[rows].astype(np.float64), ref, bf16_out=True)


@pytest.mark.slow
def test_full_size_fc1_int4_sampled(bq):
    """The FLUX-like fc1 layer in INT4 g64 at full size (M=4608, K=3072,
    N=12288, r=128), weights quantized by the library: codes and scales
    bit-exact, Y on sampled rows."""
    shape = WL.FC1_INT4
    layer = C.oracle_layer(shape)
    x = F.bf16_from_bits(layer["x_bits"])
    X = C.bf16_tensor(layer["x_bits"])
    si = C.f32_tensor(layer["smooth_inv"])
    L1s = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si)
    wc, ws, _ = bq.svdq_quantize_act(C.bf16_tensor(F.bf16_bits(layer["R"])), None, None, fmt="int4")
    codes, scales, xl1 = bq.svdq_quantize_act(X, L1s, si, fmt="int4")
    y = bq.svdq_w4a4_linear(codes, scales, xl1, wc, ws, C.bf16_tensor(F.bf16_bits(layer["L2"])),
                            C.bf16_tensor(layer["bias_bits"]), M=shape.M, N_=shape.N, K=shape.K,
                            fmt="int4")
    assert bq.svdq_check_device_status() == 0
    assert np.array_equal(wc.cpu().numpy(), C.tiled_codes("int4", layer["w_codes"]))
    assert np.array_equal(ws.cpu().numpy(), C.tiled_scales("int4", layer["w_scales"]))
    xhat = S.smooth(x, layer["smooth_inv"])
    q, sc = S.quantize_int4(xhat)
    assert np.array_equal(codes.cpu().numpy(), C.tiled_codes("int4", q))
    assert np.array_equal(scales.cpu().numpy(), C.tiled_scales("int4", sc))
    rows = np.unique(np.concatenate([np.arange(0, shape.M, 131), [shape.M - 1]]))
    ref = S.w4a4_linear(S.dequant("int4", q[rows], sc[rows]),
                        S.dequant("int4", layer["w_codes"], layer["w_scales"]),
                        S.down_proj(xhat[rows], layer["L1"]), layer["L2"],
                        F.bf16_from_bits(layer["bias_bits"]))
    C.assert_gemm_close(y.float().cpu().numpy()[rows].astype(np.float64), ref, bf16_out=True)
