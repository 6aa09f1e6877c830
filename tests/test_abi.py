"""The C-ABI library: it builds, loads, exports every call include/svdq.h
declares, and its host-side argument checks work without a GPU (no call here
reaches a kernel launch)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from bit_quantized_diffusion_b200 import _native, build
    build.build()
    return _native.load()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "svdq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([a-z_0-9]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_every_declared_call_is_exported(lib):
    from bit_quantized_diffusion_b200 import _native
    declared = _declared_functions()
    assert set(declared) == set(_native.EXPORTS), declared
    for name in declared:
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.svdq_version() == 100
    for s in range(6):
        assert lib.svdq_status_str(s)
    assert lib.svdq_status_str(5).decode().startswith("a kernel")


def test_buffer_sizes_match_the_oracle_layouts(lib):
    from oracle import layout as LO
    assert lib.svdq_codes_bytes(0, 300, 640) == 300 * 320
    assert lib.svdq_scales_bytes(0, 300, 640) == LO.nvfp4_scales_bytes(300, 640)
    assert lib.svdq_scales_bytes(1, 300, 640) == LO.int4_scales_elems(300, 640) * 2
    assert lib.awq_qweight_bytes(40, 192) == LO.awq_qweight_bytes(40, 192)
    assert lib.awq_sz_bytes(40, 192) == 48 * 3 * 4
    assert lib.svdq_codes_bytes(0, 10, 100) == 0      # K not a multiple of 64
    assert lib.svdq_scales_bytes(2, 10, 64) == 0      # unknown format


def test_argument_errors_are_caught_on_the_host(lib):
    P = ctypes.c_void_p
    good = P(0x10000)
    odd = P(0x10008)
    q = lib.svdq_quantize_act
    # M < 1, K % 64, rank 8, missing L1 for r > 0, misaligned X
    assert q(0, 0, 64, 0, good, 64, None, None, good, good, None, None) == 1
    assert q(0, 4, 100, 0, good, 100, None, None, good, good, None, None) == 1
    assert q(0, 4, 64, 8, good, 64, None, good, good, good, good, None) == 1
    assert q(0, 4, 64, 16, good, 64, None, None, good, good, good, None) == 1
    assert q(0, 4, 64, 0, odd, 64, None, None, good, good, None, None) == 2
    assert q(7, 4, 64, 0, good, 64, None, None, good, good, None, None) == 1
    g = lib.svdq_w4a4_linear
    assert g(0, 4, 40, 64, 0, good, good, None, good, good, None, None, good, 40, 0, None) == 1
    assert g(0, 4, 48, 64, 0, good, good, None, good, good, None, None, good, 44, 0, None) == 1
    assert g(0, 4, 48, 64, 0, good, good, None, good, good, None, None, good, 52, 0, None) == 2
    assert g(0, 4, 48, 64, 16, good, good, None, good, good, good, None, good, 48, 0, None) == 1
    assert g(0, 4, 48, 64, 0, good, good, None, good, good, None, None, good, 48, 3, None) == 1
    # the fused QKV epilogue: N a multiple of 384, eps finite and >= 0, both tables or
    # neither, 4-byte aligned tables, 2-byte aligned head weights
    qk = lib.svdq_w4a4_linear_qkv_norm_rope
    eps = ctypes.c_float

    def qkv(N, e=1e-6, cos=None, sin=None, norm_q=None):
        return qk(4, N, 64, 0, good, good, None, good, good, None, None, norm_q, None, eps(e), cos,
                  sin, good, N, 0, None)

    assert qkv(385) == 1 and qkv(256) == 1 and qkv(0) == 1
    assert qkv(384, -1.0) == 1 and qkv(384, float("inf")) == 1 and qkv(384, float("nan")) == 1
    assert qkv(384, cos=good) == 1 and qkv(384, sin=good) == 1
    assert qkv(384, cos=P(0x10002), sin=good) == 2 and qkv(384, cos=good, sin=P(0x10002)) == 2
    assert qkv(384, norm_q=P(0x10001)) == 2
    a = lib.awq_w4a16_linear
    assert a(0, 16, 64, 64, good, good, good, None, good, None) == 1     # M >= 1 (any M above)
    assert a(4, 16, 96, 64, good, good, good, None, good, None) == 1     # K % 64
    assert a(4, 16, 64, 32, good, good, good, None, good, None) == 1
    assert a(4, 16, 64, 64, odd, good, good, None, good, None) == 2
    assert lib.svdq_pack(0, 0, 10, 64, good, good, good, good, good, None) == 1  # zeros for ACT
    assert lib.svdq_pack(2, 0, 10, 64, good, good, None, good, good, None) == 1  # no zeros for AWQ
    assert lib.svdq_debug_wait_timeout(0, None) == 1


def test_xl1_splits_is_a_pure_function_of_the_shape(lib):
    # ceil(M/128) row blocks times S stays within 148 SMs; S a power of two <= 8, <= K/64
    assert lib.svdq_xl1_splits(4608, 3072, 32) == 4      # 36 row blocks -> 144 CTAs
    assert lib.svdq_xl1_splits(18432, 3072, 32) == 1     # 144 row blocks
    assert lib.svdq_xl1_splits(256, 512, 16) == 8        # 2 row blocks, K/64 = 8
    assert lib.svdq_xl1_splits(256, 128, 16) == 2        # K/64 = 2 caps it
    assert lib.svdq_xl1_splits(4608, 3072, 0) == 1       # no low-rank branch
    assert lib.svdq_xl1_splits(4608, 3000, 32) == 0      # K not a multiple of 64
    assert lib.svdq_xl1_splits(4608, 3072, 24) == 0      # rank not a multiple of 16


def test_binding_takes_the_rotary_tables_angle_major(lib):
    """The fused QKV call's cos/sin tables are [64, M] (angle i of row m at
    i * M + m); the binding refuses row-major [M, 64] tables before any device
    work, whatever M is."""
    import torch
    import bit_quantized_diffusion_b200 as bq
    M, N, K = 100, 384, 128
    codes = torch.zeros(M * K // 2, dtype=torch.uint8)
    scales = torch.zeros(M * K // 16, dtype=torch.uint8)
    wc = torch.zeros(N * K // 2, dtype=torch.uint8)
    ws = torch.zeros(N * K // 16, dtype=torch.uint8)
    for shape in ((M, 64), (64, M + 1), (64 * M,)):
        t = torch.zeros(shape, dtype=torch.float32)
        with pytest.raises(ValueError, match="angle-major"):
            bq.svdq_w4a4_linear_qkv_norm_rope(codes, scales, None, wc, ws, None, None, None, None, t, t,
                                              M, N, K)
