"""Pins for the oracle's quantizer, packing, tiled layouts and GEMM, against
hand-worked examples, closed forms, invariants and brute force."""

import os

import numpy as np
import pytest

from oracle import formats as F
from oracle import layout as L
from oracle import svdq as S


def _groups(golden_dir):
    out, cur = [], {}
    for line in open(os.path.join(golden_dir, "nvfp4_groups.txt")):
        line = line.split("#")[0].split()
        if not line:
            continue
        assert line[0] == "group"
        if line[1] == "xhat":
            cur = {"xhat": np.array([float(v) for v in line[2:]])}
        elif line[1] == "scale":
            cur["scale"] = int(line[2], 16)
        else:
            cur["codes"] = np.array([int(v, 16) for v in line[2:]], dtype=np.uint8)
            out.append(cur)
    return out


def test_nvfp4_hand_worked_groups(golden_dir):
    groups = _groups(golden_dir)
    assert len(groups) == 4
    xhat = np.stack([g["xhat"] for g in groups]).reshape(1, -1)
    codes, scales = S.quantize_nvfp4(xhat)
    assert scales.tolist() == [[g["scale"] for g in groups]]
    assert np.array_equal(codes.reshape(4, 16), np.stack([g["codes"] for g in groups]))


def _exact_nvfp4_operand(rng, rows, K):
    """Values exactly on the NVFP4 grid: code * 2^e with a +-6 in every group,
    so the scale is exactly 2^e and quantization must be lossless."""
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    codes[:, ::16] = rng.choice([7, 15], size=(rows, K // 16))
    e = rng.integers(-6, 8, size=(rows, K // 16))
    vals = F.e2m1_decode(codes) * np.repeat(2.0 ** e, 16, axis=1)
    return codes, e, vals


def test_nvfp4_round_trip_exact_values():
    rng = np.random.default_rng(1)
    codes, e, vals = _exact_nvfp4_operand(rng, 33, 256)
    q, s = S.quantize_nvfp4(vals)
    assert np.array_equal(F.ue4m3_decode(s), 2.0 ** e)
    # +0 and -0 dequantize alike; compare values, and codes where nonzero
    assert np.array_equal(F.e2m1_decode(q), F.e2m1_decode(codes))
    nz = (codes & 7) != 0
    assert np.array_equal(q[nz], codes[nz])
    assert np.array_equal(S.dequant_nvfp4(q, s), vals)


def test_nvfp4_power_of_two_scaling_invariance():
    rng = np.random.default_rng(2)
    x = S.smooth(rng.standard_normal((16, 128)), None)
    x = F.rn32(x)
    q0, s0 = S.quantize_nvfp4(x)
    for k in (-3, 1, 4):
        qk, sk = S.quantize_nvfp4(x * 2.0 ** k)
        assert np.array_equal(qk, q0)
        assert np.array_equal(F.ue4m3_decode(sk), F.ue4m3_decode(s0) * 2.0 ** k)


def test_nvfp4_error_bound_and_scale_choice():
    """Every element is within half a grid step (times s) of its dequantized
    value, or saturated at 6 s; the scale is the E4M3 value nearest amax/6."""
    rng = np.random.default_rng(4)
    x = F.rn32(rng.standard_normal((64, 256)) * 3)
    q, s = S.quantize_nvfp4(x)
    sv = np.repeat(F.ue4m3_decode(s), 16, axis=1)
    deq = S.dequant_nvfp4(q, s)
    step = np.where(np.abs(deq) < 2 * sv, 0.5, np.where(np.abs(deq) < 4 * sv, 1.0, 2.0)) * sv
    ok = (np.abs(deq - x) <= step / 2 * (1 + 1e-6)) | (np.abs(deq) == 6 * sv)
    assert ok.all()
    amax = np.abs(x.reshape(64, 16, 16)).max(axis=2)
    cand = F.UE4M3_VALUES
    nearest = cand[np.argmin(np.abs(cand[None, None, :] - amax[:, :, None] / 6), axis=2)]
    assert np.allclose(F.ue4m3_decode(s), nearest, rtol=0, atol=0)


def test_int4_hand_worked_group():
    x = np.zeros((1, 64))
    x[0, :10] = [7.0, -7.0, 2.5, 3.5, -2.5, 0.5, 1.5, 6.4, -0.49, -6.6]
    q, s = S.quantize_int4(x)
    assert s.tolist() == [[1.0]]        # amax 7 -> 7/7 = 1 exactly
    assert q[0, :10].tolist() == [7, -7, 2, 4, -2, 0, 2, 6, 0, -7]
    assert not q[0, 10:].any()
    # amax 10: 10/7 = 1.42857.. -> fp16 1463/1024; 1/s = 0.69993..; 10 -> 7, -5 -> -3
    y = np.zeros((1, 64))
    y[0, :3] = [10.0, -5.0, 5.0]
    q, s = S.quantize_int4(y)
    assert s[0, 0] == 1463 / 1024
    assert q[0, :3].tolist() == [7, -3, 3]


def test_int4_zero_and_round_trip():
    q, s = S.quantize_int4(np.zeros((2, 128)))
    assert not q.any() and not s.any()
    rng = np.random.default_rng(5)
    codes = rng.integers(-7, 8, size=(8, 128))
    codes[:, ::64] = 7
    e = rng.integers(-10, 5, size=(8, 2))
    vals = codes * np.repeat(2.0 ** e, 64, axis=1)
    q, s = S.quantize_int4(vals)
    assert np.array_equal(q, codes) and np.array_equal(s, 2.0 ** e)


def test_pack_nibble_order():
    assert S.pack_nibbles(np.array([[1, 2, 3, 4]])).tolist() == [[0x21, 0x43]]
    assert S.pack_nibbles(np.array([[-1, 7, -7, 0]], dtype=np.int8)).tolist() == [[0x7F, 0x09]]
    assert S.unpack_nibbles(np.array([[0x7F, 0x09]]), signed=True).tolist() == [[-1, 7, -7, 0]]
    rng = np.random.default_rng(6)
    c = rng.integers(0, 16, size=(5, 64)).astype(np.uint8)
    assert np.array_equal(S.unpack_nibbles(S.pack_nibbles(c)), c)


def test_nvfp4_scale_atom_positions():
    assert L.nvfp4_scale_offset(0, 0, 256) == 0
    assert L.nvfp4_scale_offset(33, 5, 256) == 512 + 16 + 4 + 1
    assert L.nvfp4_scale_offset(130, 0, 128) == 2 * 512 + 2 * 16
    assert L.nvfp4_scale_offset(127, 3, 64) == 31 * 16 + 3 * 4 + 3
    rng = np.random.default_rng(7)
    s = rng.integers(0, 127, size=(200, 24)).astype(np.uint8)
    t = L.tile_nvfp4_scales(s)
    assert t.size == 256 * 24
    assert np.array_equal(L.untile_nvfp4_scales(t, 200, 384), s)
    # padding rows hold zeros, and every byte is written exactly once
    m, j = np.meshgrid(np.arange(256), np.arange(24), indexing="ij")
    offs = L.nvfp4_scale_offset(m, j, 384)
    assert np.unique(offs).size == offs.size == t.size
    assert not t[L.nvfp4_scale_offset(m[200:], j[200:], 384)].any()


def test_int4_code_tiling_hand_bytes():
    # values (element 2j low nibble), two's complement: (1, -1) -> 0xF1,
    # (-7, 7) -> 0x79, (0, -3) -> 0xD0
    q = np.array([[1, -1, -7, 7, 0, -3]])
    t = L.tile_int4_codes(q)
    assert t.tolist() == [[0xF1, 0x79, 0xD0]]
    assert np.array_equal(L.untile_int4_codes(t), q)
    # the plain form holds the same bytes
    assert S.pack_nibbles(q).tolist() == [[0xF1, 0x79, 0xD0]]
    every = np.arange(-7, 8).repeat(2).reshape(1, -1)
    assert np.array_equal(L.untile_int4_codes(L.tile_int4_codes(every)), every)


def test_int4_scale_tiling():
    s = np.arange(6 * 3, dtype=np.float64).reshape(6, 3) / 8
    t = L.tile_int4_scales(s)
    assert t.size == 3 * 128
    assert t.view(np.float16)[128 + 2] == s[2, 1]
    assert np.array_equal(L.untile_int4_scales(t, 6, 192), s)


def test_awq_fragment_tiling_hand_word():
    n, k = np.meshgrid(np.arange(16), np.arange(64), indexing="ij")
    q = ((n + k) % 16).astype(np.uint8)
    t = L.tile_awq_qweight(q)
    w = t.view(np.uint32).reshape(32, 4)[5, 1]       # lane 5: r0 = 1, c0 = 2; j = 1
    vals = [3, 11, 11, 3, 4, 12, 12, 4]
    assert w == sum(v << (4 * i) for i, v in enumerate(vals))
    rng = np.random.default_rng(8)
    q2 = rng.integers(0, 16, size=(40, 192)).astype(np.uint8)
    assert np.array_equal(L.untile_awq_qweight(L.tile_awq_qweight(q2), 40, 192), q2)


def test_awq_sz_tiling():
    rng = np.random.default_rng(9)
    s = rng.integers(0, 65535, size=(20, 3)).astype(np.uint16)
    z = rng.integers(0, 65535, size=(20, 3)).astype(np.uint16)
    t = L.tile_awq_sz(s, z)
    assert t.size == 32 * 3 * 2
    assert t[((1 * 3 + 2) * 16 + 3) * 2] == s[19, 2]
    s2, z2 = L.untile_awq_sz(t, 20, 192)
    assert np.array_equal(s2, s) and np.array_equal(z2, z)


def test_w4a4_exact_closed_form():
    """With both operands exactly on the NVFP4 grid, the 4-bit GEMM is lossless:
    Y equals the plain product of the dense matrices, plus the low-rank term."""
    rng = np.random.default_rng(10)
    M, N, K, r = 40, 24, 128, 16
    _, _, xa = _exact_nvfp4_operand(rng, M, K)
    _, _, wr = _exact_nvfp4_operand(rng, N, K)
    L1 = rng.integers(-3, 4, size=(K, r)).astype(np.float64)
    L2 = rng.integers(-3, 4, size=(r, N)).astype(np.float64)
    b = rng.integers(-5, 6, size=N).astype(np.float64)
    qa, sa = S.quantize_nvfp4(xa)
    qw, sw = S.quantize_nvfp4(wr)
    xl1 = S.down_proj(xa, L1)
    y = S.w4a4_linear(S.dequant_nvfp4(qa, sa), S.dequant_nvfp4(qw, sw), xl1, L2, b)
    want = xa @ wr.T + (xa @ L1) @ L2 + b
    assert np.array_equal(y, want)


def test_w4a4_brute_force_small():
    rng = np.random.default_rng(11)
    M, N, K, r = 3, 5, 64, 2
    x = F.rn32(rng.standard_normal((M, K)))
    w = F.rn32(rng.standard_normal((N, K)) * 0.1)
    qa, sa = S.quantize_nvfp4(x)
    qw, sw = S.quantize_nvfp4(w)
    L1 = F.bf16_round(rng.standard_normal((K, r)))
    L2 = F.bf16_round(rng.standard_normal((r, N)))
    b = F.bf16_round(rng.standard_normal(N))
    y = S.w4a4_linear(S.dequant_nvfp4(qa, sa), S.dequant_nvfp4(qw, sw),
                      S.down_proj(x, L1), L2, b)
    ev, sv = F.e2m1_decode, F.ue4m3_decode
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += (float(ev(qa[m, k])) * float(sv(sa[m, k // 16]))
                        * float(ev(qw[n, k])) * float(sv(sw[n, k // 16])))
            for j in range(r):
                acc += sum(x[m, k] * L1[k, j] for k in range(K)) * L2[j, n]
            acc += b[n]
            assert abs(acc - y[m, n]) <= 1e-9 * max(1.0, abs(acc))


def test_w4a4_rank_zero_and_zero_residual():
    rng = np.random.default_rng(12)
    M, N, K, r = 16, 8, 64, 16
    x = F.rn32(rng.standard_normal((M, K)))
    L1 = F.bf16_round(rng.standard_normal((K, r)))
    L2 = F.bf16_round(rng.standard_normal((r, N)))
    qa, sa = S.quantize_nvfp4(x)
    a = S.dequant_nvfp4(qa, sa)
    # zero residual: the 4-bit term vanishes and Y is the low-rank branch
    qz, sz = S.quantize_nvfp4(np.zeros((N, K)))
    assert not qz.any() and not sz.any()
    y = S.w4a4_linear(a, S.dequant_nvfp4(qz, sz), S.down_proj(x, L1), L2, None)
    assert np.allclose(y, (x @ L1) @ L2, rtol=1e-12, atol=1e-12)
    # rank zero: Y is the plain dequantized product
    w = F.rn32(rng.standard_normal((N, K)))
    qw, sw = S.quantize_nvfp4(w)
    y0 = S.w4a4_linear(a, S.dequant_nvfp4(qw, sw), None, np.zeros((0, N)), None)
    assert np.array_equal(y0, a @ S.dequant_nvfp4(qw, sw).T)


def test_row_permutation_equivariance():
    rng = np.random.default_rng(13)
    x_bits = (rng.standard_normal((32, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    w = F.rn32(rng.standard_normal((8, 128)) * 0.1)
    qw, sw = S.quantize_nvfp4(w)
    L1 = F.bf16_round(rng.standard_normal((128, 16)))
    L2 = F.bf16_round(rng.standard_normal((16, 8)))
    si = F.rn32(rng.uniform(0.5, 2.0, 128))
    perm = rng.permutation(32)
    y = S.svdq_forward("nvfp4", x_bits, si, L1, L2, qw, sw)["Y"]
    yp = S.svdq_forward("nvfp4", x_bits[perm], si, L1, L2, qw, sw)["Y"]
    assert np.array_equal(yp, y[perm])


def test_smoothing_is_one_float32_multiply():
    x = np.array([[1.0, 3.0]])
    si = np.array([F.rn32(1 / 3.0)[()], 0.5])
    xh = S.smooth(x, si)
    assert xh[0, 0] == float(np.float32(1.0) * np.float32(1 / 3.0))
    assert xh[0, 1] == 1.5


def test_lowrank_operand_split():
    """hi + lo carries smooth_inv * L1 to about 2^-17 relative; both are bf16;
    without smoothing the lo plane is zero. Summed, the split down-projection
    X (hi + lo) equals x_hat L1 within that bound."""
    rng = np.random.default_rng(14)
    K, r = 128, 16
    L1 = F.bf16_round(rng.standard_normal((K, r)))
    si = F.rn32(rng.uniform(0.1, 3.0, K))
    op = L.lowrank_operand(L1, si)
    assert op.shape == (2, r, K)
    assert np.array_equal(F.bf16_round(op), op)
    v = F.rn32(L1.T * si[None, :])
    assert np.all(np.abs(op[0] + op[1] - v) <= np.abs(v) * 2.0 ** -17)
    plain = L.lowrank_operand(L1, None)
    assert np.array_equal(plain[0], L1.T) and not plain[1].any()
    x = F.bf16_round(rng.standard_normal((8, K)))
    xhat = S.smooth(x, si)
    ref = S.down_proj(xhat, L1)
    got = x @ (op[0] + op[1]).T
    assert np.all(np.abs(got - ref) <= (np.abs(xhat) @ np.abs(L1)) * 2.0 ** -16)
