"""The AWQ W4A16 linear on the tensor cores (awq_gemm_kernel, through
awq_w4a16_linear) against the oracle's AWQ linear, which forms every weight
(q - z) s exactly in float64: token counts above the GEMV's 64 (one and several
128-token tiles, ragged token tails), weight rows that end inside a 128-row
tile and inside a 16-row block, one to many 64-wide groups, with and without
bias; the same kernel forced at small token counts (16-token tiles, 16- and
32-column epilogue slices); and the adaLN projection's full width at 256 tokens
and at its own 4 tokens, where the two kernels are also compared with each other."""

import os

import numpy as np
import pytest

import workloads as WL
from oracle import awq as OA
from oracle import formats as F
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


class forced_path:
    """SVDQ_AWQ_PATH for the calls inside the block (the library reads it per call)."""

    def __init__(self, value):
        self.value = value

    def __enter__(self):
        self.old = os.environ.get("SVDQ_AWQ_PATH")
        if self.value is None:
            os.environ.pop("SVDQ_AWQ_PATH", None)
        else:
            os.environ["SVDQ_AWQ_PATH"] = self.value

    def __exit__(self, *exc):
        if self.old is None:
            os.environ.pop("SVDQ_AWQ_PATH", None)
        else:
            os.environ["SVDQ_AWQ_PATH"] = self.old


def _packed(bq, q, s, z):
    Nn, K = q.shape
    return bq.svdq_pack("awq", "nvfp4", Nn, K, C.u8_tensor(S.pack_nibbles(q).reshape(-1)),
                        C.u8_tensor(F.bf16_bits(s).view(np.uint8).reshape(-1)),
                        C.u8_tensor(F.bf16_bits(z).view(np.uint8).reshape(-1)))


def _case(M, Nn, K, seed, bias=True):
    rng = np.random.default_rng(seed)
    x_bits = WL.to_bf16_bits(rng.standard_normal((M, K)))
    w = F.bf16_round(rng.standard_normal((Nn, K)) * 0.02)
    q, s, z = OA.quantize_weight(w)
    b_bits = WL.to_bf16_bits(rng.standard_normal(Nn) * 0.1) if bias else None
    ref = OA.linear(F.bf16_from_bits(x_bits), q, s, z,
                    F.bf16_from_bits(b_bits) if bias else None)
    return x_bits, q, s, z, b_bits, ref


def _run(bq, x_bits, q, s, z, b_bits, path):
    qt, szt = _packed(bq, q, s, z)
    with forced_path(path):
        y = bq.awq_w4a16_linear(C.bf16_tensor(x_bits), qt, szt,
                                C.bf16_tensor(b_bits) if b_bits is not None else None, q.shape[0])
    assert bq.svdq_check_device_status() == 0
    return y.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M,Nn,K,bias", [
    (65, 256, 128, True),     # just above the GEMV's range: one 80-token tile
    (100, 272, 640, True),    # rows end inside a 16-row block of the third 128-row tile
    (128, 128, 64, False),    # one full tile, a single group, no bias
    (129, 384, 256, True),    # two token tiles, the second with one token
    (300, 208, 1024, True),   # three token tiles, ragged rows
])
def test_awq_tensor_core_path_matches_the_oracle(bq, M, Nn, K, bias):
    x_bits, q, s, z, b_bits, ref = _case(M, Nn, K, 700 + M + Nn, bias)
    y = _run(bq, x_bits, q, s, z, b_bits, None)  # M > 64 takes the tensor cores by itself
    C.assert_gemm_close(y, ref, bf16_out=True, what="AWQ tensor-core Y")


@pytest.mark.parametrize("M,Nn,K", [(1, 64, 128), (4, 272, 640), (13, 96, 256), (16, 160, 192),
                                    (33, 128, 512), (64, 48, 128)])
def test_awq_tensor_core_path_forced_at_small_m(bq, M, Nn, K):
    x_bits, q, s, z, b_bits, ref = _case(M, Nn, K, 800 + M)
    y = _run(bq, x_bits, q, s, z, b_bits, "1")
    C.assert_gemm_close(y, ref, bf16_out=True, what="AWQ tensor-core Y (forced)")


def test_awq_adaln_width_at_256_tokens(bq):
    shape = WL.AWQ_MOD
    d = WL.awq_inputs(shape)
    q, s, z = OA.quantize_weight(F.bf16_from_bits(d["W"]))
    rng = np.random.default_rng(900)
    x_bits = WL.to_bf16_bits(rng.standard_normal((256, shape.K)))
    ref = OA.linear(F.bf16_from_bits(x_bits), q, s, z, F.bf16_from_bits(d["bias"]))
    y = _run(bq, x_bits, q, s, z, d["bias"], None)
    C.assert_gemm_close(y, ref, bf16_out=True, what="AWQ adaLN width, 256 tokens")


def test_awq_adaln_both_kernels_at_4_tokens(bq):
    """The adaLN projection as the bench runs it (M = 4): both kernels within the
    tolerance of the oracle; their outputs differ only by float32 summation order."""
    shape = WL.AWQ_MOD
    d = WL.awq_inputs(shape)
    q, s, z = OA.quantize_weight(F.bf16_from_bits(d["W"]))
    ref = OA.linear(F.bf16_from_bits(d["X"]), q, s, z, F.bf16_from_bits(d["bias"]))
    y_gemv = _run(bq, d["X"], q, s, z, d["bias"], "0")
    y_tc = _run(bq, d["X"], q, s, z, d["bias"], "1")
    C.assert_gemm_close(y_gemv, ref, bf16_out=True, what="AWQ adaLN Y (GEMV)")
    C.assert_gemm_close(y_tc, ref, bf16_out=True, what="AWQ adaLN Y (tensor cores)")


def test_forcing_the_gemv_above_its_range_is_refused(bq):
    x_bits, q, s, z, b_bits, _ = _case(65, 64, 64, 999)
    qt, szt = _packed(bq, q, s, z)
    with forced_path("0"), pytest.raises(bq.SvdqError) as e:
        bq.awq_w4a16_linear(C.bf16_tensor(x_bits), qt, szt, None, 64)
    assert e.value.status == 3
