"""Seeded random shapes through the same checks as the fixed-shape parity tests:
the quantizer's codes and scales bit-exact and the W4A4 linear within the
stated tolerance of the oracle (both formats, M from 1 row to several tiles,
any N % 16, K % 64 and r % 16 within the supported ranges), the fused QKV
projection, the AWQ linear on either of its kernels, and the fused MLP. The
shapes are drawn once from a fixed seed, so a failure names a reproducible case."""

import numpy as np
import pytest

import workloads as WL
from tests import svdq_cases as C
from tests import test_gpu_awq_gemm as TA
from tests import test_gpu_mlp as TM
from tests import test_gpu_parity as TP
from tests import test_gpu_qkv_epilogue as TQ

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

_rng = np.random.default_rng(20260)
GEMM = [(str(_rng.choice(["nvfp4", "int4"])), int(_rng.integers(1, 700)), int(_rng.integers(1, 33)) * 64,
         int(_rng.integers(1, 64)) * 16, int(_rng.choice([0, 16, 32, 48, 64, 128])), bool(_rng.integers(0, 2)))
        for _ in range(16)]
# at least two INT4 cases of at most 128 rows and more than 128 columns
GEMM += [("int4", 37, 448, 336, 32, True), ("int4", 128, 192, 144, 0, False)]
QKV = [(int(_rng.integers(1, 900)), int(_rng.integers(1, 5)), int(_rng.integers(1, 17)) * 64,
        int(_rng.choice([0, 16, 32, 64])), bool(_rng.integers(0, 2)), bool(_rng.integers(0, 2)),
        bool(_rng.integers(0, 2))) for _ in range(6)]
AWQ = [(int(_rng.integers(1, 300)), int(_rng.integers(1, 40)) * 16, int(_rng.integers(1, 17)) * 64,
        bool(_rng.integers(0, 2))) for _ in range(6)]
# fused MLP: N1 % 128, r2 in {0, 32, 64, 96, 128} and at most fc2's width N2
MLP = []
while len(MLP) < 5:
    _m = (int(_rng.integers(1, 1500)), int(_rng.integers(1, 17)) * 64, int(_rng.integers(1, 13)) * 128,
          int(_rng.integers(1, 33)) * 16, int(_rng.choice([0, 16, 32, 64])), int(_rng.choice([0, 32, 64, 96, 128])))
    if _m[5] <= _m[3]:
        MLP.append(_m)


@pytest.fixture(scope="module")
def bq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_quantized_diffusion_b200 as bq
    return bq


@pytest.mark.parametrize("fmt,M,K,N,r,bias", GEMM, ids=lambda v: str(v))
def test_random_w4a4_layer(bq, fmt, M, K, N, r, bias):
    shape = WL.custom_svdq(f"rand_{fmt}_{M}_{K}_{N}_{r}", M, K, N, r, fmt=fmt, seed=M + K + N + r)
    TP.test_quantize_act_matches_oracle(bq, shape)
    TP.test_w4a4_linear_matches_oracle(bq, shape, bias)


@pytest.mark.parametrize("M,H,K,r,out_f32,weights,rope", QKV, ids=lambda v: str(v))
def test_random_fused_qkv(bq, M, H, K, r, out_f32, weights, rope):
    TQ.test_fused_qkv_matches_the_oracle(bq, M, H, K, r, out_f32, weights, rope)


@pytest.mark.parametrize("M,N,K,bias", AWQ, ids=lambda v: str(v))
def test_random_awq(bq, M, N, K, bias):
    x_bits, q, s, z, b_bits, ref = TA._case(M, N, K, 9000 + M + N, bias)
    y = TA._run(bq, x_bits, q, s, z, b_bits, None)
    C.assert_gemm_close(y, ref, bf16_out=True, what="AWQ Y")


@pytest.mark.parametrize("M,K1,N1,N2,r1,r2", MLP, ids=lambda v: str(v))
def test_random_fused_mlp(bq, M, K1, N1, N2, r1, r2):
    d1, p1, d2, p2 = TM._layers(M, K1, N1, N2, r1, r2, seed=7000 + M)
    out = TM._run(bq, d1, p1, d2, p2, M, K1, N1, N2, r1, r2)
    TM._check(bq, out, d1, p1, d2, p2, M, r2)
