"""Full-size parity of the workload configurations that the smaller parity
cases only mirror in structure: the FLUX-like MLP pair (fc1 3072 -> 12288 and
fc2 12288 -> 3072, r = 128), the rank sweep at hidden 3840 (N = 3840 and
15360, r in {0, 32, 128, 256}), the 4 x 4608-token batch (M = 18432, where K
is not split) and the adaLN AWQ projection (M = 4, N = 18432).

Each layer runs at its full size through the C ABI in the launch configuration
the library picks for it (the same the benchmark times). The oracle checks, on
a sample of rows it can afford (every row of a spread of 128-row blocks, plus
the last row): activation codes and scales bit-exact, the weight quantizer's
codes and scales bit-exact over the whole weight, xl1 within its stated bound,
and Y against the unrounded float64 layer with the stated tolerances. The AWQ
projection is checked on every output.
"""

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
pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def bq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_quantized_diffusion_b200 as bq
    return bq


def sample_rows(M: int, n_blocks: int = 6) -> np.ndarray:
    """Whole 128-row blocks spread over M (first, last and evenly between), so
    every position inside a block and the ragged tail are covered."""
    blocks = max(1, (M + 127) // 128)
    picks = np.unique(np.linspace(0, blocks - 1, min(n_blocks, blocks)).round().astype(int))
    rows = np.concatenate([np.arange(b * 128, min(M, b * 128 + 128)) for b in picks])
    return np.unique(np.concatenate([rows, [M - 1]]))


def layers_sharing_svd(shapes):
    """Oracle prep for layers that differ only in rank: one float64 SVD of the
    smoothed weight, each rank taking its leading factors (the SVD split's
    columns depend only on their own singular triple), then the residual and
    its quantization per rank, as the oracle's prepare_svdq_layer does."""
    base = shapes[0]
    assert all((s.M, s.K, s.N, s.seed, s.fmt) == (base.M, base.K, base.N, base.seed, base.fmt)
               for s in shapes)
    d = WL.svdq_inputs(base)
    x = F.bf16_from_bits(d["X"])
    w = F.bf16_from_bits(d["W"])
    lam, smooth_inv = P.smoothing_factors(x, w)
    w_hat = w * (1.0 / smooth_inv)[None, :]
    r_max = max(s.r for s in shapes)
    L1_all, L2_all = P.svd_split(w_hat, r_max)
    out = []
    for s in shapes:
        L1, L2 = L1_all[:, :s.r], L2_all[:s.r]
        R = F.bf16_round(w_hat - (L1 @ L2).T)
        w_codes, w_scales = S.quantize(s.fmt, R)
        out.append({"shape": s, "x_bits": d["X"], "w_bits": d["W"], "bias_bits": d["bias"],
                    "lambda": lam, "smooth_inv": smooth_inv, "L1": L1, "L2": L2, "R": R,
                    "w_codes": w_codes, "w_scales": w_scales})
    return out


def check_layer(bq, layer, rows: np.ndarray):
    shape = layer["shape"]
    M, K, N, r = shape.M, shape.K, shape.N, shape.r
    assert shape.fmt == "nvfp4"
    x = F.bf16_from_bits(layer["x_bits"])
    X = C.bf16_tensor(layer["x_bits"])
    si = C.f32_tensor(layer["smooth_inv"])
    L1s = bq.svdq_pack_lowrank(C.bf16_tensor(F.bf16_bits(layer["L1"])), si) if r else None
    wc, ws, _ = bq.svdq_quantize_act(C.bf16_tensor(F.bf16_bits(layer["R"])), None, None)
    codes, scales, xl1 = bq.svdq_quantize_act(X, L1s, si)
    L2 = C.bf16_tensor(F.bf16_bits(layer["L2"])) if r else None
    y = bq.svdq_w4a4_linear(codes, scales, xl1, wc, ws, L2, C.bf16_tensor(layer["bias_bits"]),
                            M=M, N_=N, K=K)
    assert bq.svdq_check_device_status() == 0
    # the weight quantizer, over the whole residual
    assert np.array_equal(wc.cpu().numpy(), S.pack_nibbles(layer["w_codes"]).reshape(-1))
    assert np.array_equal(ws.cpu().numpy(), LO.tile_nvfp4_scales(layer["w_scales"]))
    # activations on the sampled rows
    xhat = S.smooth(x[rows], layer["smooth_inv"])
    q, sc = S.quantize_nvfp4(xhat)
    got_codes = codes.cpu().numpy().reshape(M, K // 2)[rows]
    assert np.array_equal(got_codes, S.pack_nibbles(q))
    got_scales = LO.untile_nvfp4_scales(scales.cpu().numpy(), M, K)[rows]
    assert np.array_equal(got_scales, sc)
    xl1_ref = S.down_proj(xhat, layer["L1"]) if r else None
    if r:
        got_xl1 = xl1.cpu().numpy()[rows].astype(np.float64)
        assert np.all(np.abs(got_xl1 - xl1_ref) <= C.xl1_bound(xhat, layer["L1"]))
    ref = S.w4a4_linear(S.dequant_nvfp4(q, sc), S.dequant_nvfp4(layer["w_codes"], layer["w_scales"]),
                        xl1_ref, layer["L2"] if r else None, F.bf16_from_bits(layer["bias_bits"]))
    return C.assert_gemm_close(y.float().cpu().numpy()[rows].astype(np.float64), ref,
                               bf16_out=True, what=shape.name)


@pytest.mark.parametrize("shape", [WL.FC1, WL.FC2, WL.BIG], ids=lambda s: s.name)
def test_full_size_layer_sampled(bq, shape):
    layer = C.oracle_layer(shape)
    check_layer(bq, layer, sample_rows(shape.M))


@pytest.mark.parametrize("n", [3840, 15360])
def test_rank_sweep_full_size_sampled(bq, n):
    shapes = [s for s in WL.RANK_SWEEP if s.N == n]
    assert sorted(s.r for s in shapes) == [0, 32, 128, 256]
    rows = sample_rows(shapes[0].M, n_blocks=4)
    for layer in layers_sharing_svd(shapes):
        check_layer(bq, layer, rows)


def test_awq_adaln_full_size(bq):
    shape = WL.AWQ_MOD
    d = WL.awq_inputs(shape)
    q, s, z = OA.quantize_weight(F.bf16_from_bits(d["W"]))
    ref = OA.linear(F.bf16_from_bits(d["X"]), q, s, z, F.bf16_from_bits(d["bias"]))
    qt, szt = bq.svdq_pack("awq", "nvfp4", shape.N, shape.K,
                           C.u8_tensor(S.pack_nibbles(q).reshape(-1)),
                           C.u8_tensor(F.bf16_bits(s).view(np.uint8).reshape(-1)),
                           C.u8_tensor(F.bf16_bits(z).view(np.uint8).reshape(-1)))
    y = bq.awq_w4a16_linear(C.bf16_tensor(d["X"]), qt, szt, C.bf16_tensor(d["bias"]), shape.N)
    assert bq.svdq_check_device_status() == 0
    C.assert_gemm_close(y.float().cpu().numpy().astype(np.float64), ref, bf16_out=True,
                        what="AWQ adaLN Y")
