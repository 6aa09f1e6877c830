"""Host logic of the layer classes, with the library calls replaced by fakes that
record what they are given: which workspaces, shapes and scale pairs reach
which call, and which configurations are refused. No GPU and no compute."""

import pytest

torch = pytest.importorskip("torch")
import bit_quantized_diffusion_b200.layers as L  # noqa: E402

BF = torch.bfloat16


def weights(N, K, r, fmt="nvfp4", two_level=False):
    return {"smooth_inv": torch.ones(K), "L1s": torch.zeros(2, r, K, dtype=BF),
            "L2": torch.zeros(r, N, dtype=BF) if r else None,
            "w_codes": torch.zeros(N * K // 2, dtype=torch.uint8),
            "w_scales": torch.zeros(N * K // 16, dtype=torch.uint8),
            "w_tscale": torch.ones(2) if two_level else None, "fmt": fmt, "N": N, "K": K, "r": r}


class Recorder:
    def __init__(self, monkeypatch):
        self.calls = []
        rec = self

        def quant(x, L1s, si, fmt="nvfp4", codes=None, scales=None, xl1=None, stream=None):
            rec.calls.append(("quantize", x.shape[0], codes, scales, xl1))
            return codes, scales, xl1

        def quant2(x, scale, L1s, si, codes=None, scales=None, xl1=None, stream=None):
            rec.calls.append(("quantize_two_level", x.shape[0], scale, codes, xl1))
            return codes, scales, xl1

        def tscale(x, si, scale=None, stream=None):
            rec.calls.append(("tensor_scale", x.shape[0], scale))
            return scale

        def gemm(codes, scales, xl1, wc, ws, L2, bias, M, N, K, fmt="nvfp4", Y=None, stream=None):
            rec.calls.append(("linear", M, N, K, xl1))
            return "Y"

        def gemm2(codes, scales, a_t, xl1, wc, ws, w_t, L2, bias, M, N, K, Y=None, stream=None):
            rec.calls.append(("linear_two_level", M, N, K, a_t, w_t))
            return "Y"

        def qkv(codes, scales, xl1, wc, ws, L2, bias, nq, nk, cos, sin, M, N, K, eps=1e-6, Y=None,
                stream=None):
            rec.calls.append(("qkv", M, N, K, nq, nk, cos, sin, eps, xl1))
            return "Y"

        for name, fn in (("svdq_quantize_act", quant), ("svdq_quantize_act_two_level", quant2),
                         ("svdq_tensor_scale", tscale), ("svdq_w4a4_linear", gemm),
                         ("svdq_w4a4_linear_two_level", gemm2), ("svdq_w4a4_linear_qkv_norm_rope", qkv)):
            monkeypatch.setattr(L, name, fn)


def test_qkv_layer_routes_its_workspaces_and_epilogue_inputs(monkeypatch):
    rec = Recorder(monkeypatch)
    N, K, r = 3 * 2 * 128, 512, 32
    gq, gk = torch.ones(128, dtype=BF), torch.ones(128, dtype=BF)
    layer = L.SvdqQkvNormRope(weights(N, K, r), None, max_tokens=300, norm_q=gq, norm_k=gk, eps=1e-5)
    assert layer.heads == 2
    x = torch.zeros(260, K, dtype=BF)
    cos, sin = torch.zeros(64, 260), torch.zeros(64, 260)
    assert layer(x, cos, sin) == "Y"
    (q, M, codes, scales, xl1), g = rec.calls
    assert q == "quantize" and M == 260 and codes is layer.codes and scales is layer.scales
    # the down-projection's working space is the layer's own, cut to this call's splits
    assert xl1.data_ptr() == layer.xl1.data_ptr()
    assert xl1.numel() == L.svdq_xl1_splits(260, K, r) * 260 * r
    assert g[:4] == ("qkv", 260, N, K) and g[4] is gq and g[5] is gk and g[6] is cos and g[7] is sin
    assert g[8] == pytest.approx(1e-5) and g[9] is xl1
    with pytest.raises(ValueError):
        layer(torch.zeros(301, K, dtype=BF))


@pytest.mark.parametrize("N,fmt,two_level", [(3 * 128 * 2 + 16, "nvfp4", False), (768, "int4", False),
                                             (768, "nvfp4", True)])
def test_qkv_layer_refuses_what_the_call_cannot_do(N, fmt, two_level):
    with pytest.raises(ValueError):
        L.SvdqQkvNormRope(weights(N, 512, 16, fmt, two_level), None, max_tokens=64)


def test_two_level_layer_scale_pairs(monkeypatch):
    rec = Recorder(monkeypatch)
    w = weights(256, 512, 16, two_level=True)
    x = torch.zeros(100, 512, dtype=BF)
    per_call = L.SvdqW4A4Linear(w, None, max_tokens=128)
    per_call(x)
    ts, q2, g2 = rec.calls
    # no calibrated pair: the activation's pair goes into the layer's own buffer,
    # then to the quantizer and the GEMM beside the weight's pair
    assert ts[0] == "tensor_scale" and ts[2] is per_call._a_scale
    assert q2[0] == "quantize_two_level" and q2[2] is per_call._a_scale
    assert g2[0] == "linear_two_level" and g2[4] is per_call._a_scale and g2[5] is w["w_tscale"]
    rec.calls.clear()
    calibrated = torch.ones(2)
    L.SvdqW4A4Linear(w, None, max_tokens=128, act_scale=calibrated)(x)
    assert [c[0] for c in rec.calls] == ["quantize_two_level", "linear_two_level"]
    assert rec.calls[0][2] is calibrated and rec.calls[1][4] is calibrated


def test_one_level_layer(monkeypatch):
    rec = Recorder(monkeypatch)
    layer = L.SvdqW4A4Linear(weights(256, 512, 0), None, max_tokens=64)
    layer(torch.zeros(64, 512, dtype=BF))
    assert [c[0] for c in rec.calls] == ["quantize", "linear"]
    assert rec.calls[0][4] is None  # r = 0: no down-projection


def fake_prep(monkeypatch):
    seen = {}

    def prepare(w, x_absmax, rank, fmt="nvfp4", two_level=False):
        seen.update(w=w, x_absmax=x_absmax, rank=rank, fmt=fmt, two_level=two_level)
        N, K = w.shape
        return weights(N, K, rank, fmt, two_level)

    def prepare_awq(w):
        seen.update(awq=w)
        return {"qweight": None, "sz": None, "N": w.shape[0], "K": w.shape[1]}

    monkeypatch.setattr(L.prep, "prepare_svdq_weights", prepare)
    monkeypatch.setattr(L.prep, "prepare_awq_weights", prepare_awq)
    return seen


def test_from_linears_joins_q_k_v_in_order(monkeypatch):
    seen = fake_prep(monkeypatch)
    K, Hd = 512, 2 * 128
    q, k, v = (torch.full((Hd, K), float(i), dtype=BF) for i in (1, 2, 3))
    bq_, bv = torch.full((Hd,), 1.0, dtype=BF), torch.full((Hd,), 3.0, dtype=BF)
    ax = torch.ones(K)
    gq = torch.ones(128, dtype=BF)
    layer = L.SvdqQkvNormRope.from_linears(q, k, v, (bq_, None, bv), ax, 32, max_tokens=64,
                                           norm_q=gq, eps=1e-5)
    w = seen["w"]
    assert w.shape == (3 * Hd, K) and seen["rank"] == 32 and seen["x_absmax"] is ax
    assert torch.equal(w[:Hd], q) and torch.equal(w[Hd:2 * Hd], k) and torch.equal(w[2 * Hd:], v)
    # a missing bias is zero in its third of the joined bias
    assert torch.equal(layer.bias[:Hd], bq_) and not layer.bias[Hd:2 * Hd].any()
    assert torch.equal(layer.bias[2 * Hd:], bv)
    assert layer.heads == 2 and layer.norm_q is gq and layer.norm_k is None and layer.eps == 1e-5
    assert L.SvdqQkvNormRope.from_linears(q, k, v, None, ax, 0, max_tokens=8).bias is None
    with pytest.raises(ValueError):
        L.SvdqQkvNormRope.from_linears(q, k[:128], v, None, ax, 0, max_tokens=8)


def test_from_linear_constructors(monkeypatch):
    seen = fake_prep(monkeypatch)
    w = torch.zeros(256, 512, dtype=BF)
    b = torch.zeros(256, dtype=BF)
    scale = torch.ones(2)
    lin = L.SvdqW4A4Linear.from_linear(w, b, torch.ones(512), 16, max_tokens=32, two_level=True,
                                       act_scale=scale)
    assert seen["w"] is w and seen["two_level"] and lin.two_level and lin.act_scale is scale
    assert lin.bias is b and lin.r == 16
    awq = L.AwqW4A16Linear.from_linear(w, b)
    assert seen["awq"] is w and awq.bias is b and awq.w["N"] == 256
