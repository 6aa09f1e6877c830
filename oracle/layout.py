"""Tiled (kernel-side) layouts of quantized operands, defined by index formulas.

ORACLE -- test infrastructure only.

These are this library's own storage formats (the pages fix none); the CUDA
pack/unpack calls implement the same formulas independently, and the parity
tests compare the bytes.

NVFP4 scales (activations and weights), "atom" layout
    Rows are padded to a multiple of 128 with scale code 0. Scale column
    j = k // 16. Atom a = (m // 128) * (K // 64) + j // 4 holds 512 bytes;
    inside it, byte (m % 32) * 16 + ((m % 128) // 32) * 4 + (j % 4).
    So the four scales a row needs for one 64-wide K block are one 32-bit word,
    and 32 consecutive rows' words are 16 bytes apart.

INT4 scales (activations and weights), group-major
    FP16 values at [K // 64][rows padded to 128], padding 0.

NVFP4 / INT4 codes
    Plain: row-major, K contiguous, two codes per byte, element 2j in the low
    nibble (INT4 as two's complement). The tiled codes of both formats are the
    same bytes (INT4 values -7..7 as two's complement nibbles, v & 15).

AWQ qweight, MMA-fragment order
    N padded to 16 rows. For row block b = n // 16 and group g = k // 64 there
    are 512 bytes = 32 lanes x 16 bytes. Lane t (r0 = t // 4, c0 = 2 (t % 4))
    holds four 32-bit words w_j (j = 0..3 covers k = 64 g + 16 j + [0, 16)).
    Nibble slot s of w_j (bits 4s..4s+3) holds, for s = 0..7:
        W[r0][c0], W[r0+8][c0], W[r0][c0+8], W[r0+8][c0+8],
        W[r0][c0+1], W[r0+8][c0+1], W[r0][c0+9], W[r0+8][c0+9]
    (row offsets within the block, column offsets from 64 g + 16 j).
    Byte offset of w_j: ((b * (K // 64) + g) * 32 + t) * 16 + 4 j.

Down-projection operand L1s (the smoothing folded into the factor)
    v = RN32(smooth_inv[k] * L1[k, j]), hi = BF16(v), lo = BF16(RN32(v - hi));
    planes [2][r][K]: L1s[0, j, k] = hi, L1s[1, j, k] = lo.

AWQ scales and zeros, interleaved
    bf16 pairs (s, z) at [N / 16][K // 64][16 rows][2], rows padded with (0, 0).
"""

from __future__ import annotations

import numpy as np


def pad_rows(rows: int, mult: int = 128) -> int:
    return (rows + mult - 1) // mult * mult


# ------------------------------------------------------------- NVFP4 scales
def nvfp4_scale_offset(m: np.ndarray, j: np.ndarray, K: int) -> np.ndarray:
    """Byte offset of scale (row m, column j = k // 16) in the atom layout."""
    m = np.asarray(m, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    atom = (m // 128) * (K // 64) + j // 4
    return atom * 512 + (m % 32) * 16 + ((m % 128) // 32) * 4 + (j % 4)


def nvfp4_scales_bytes(rows: int, K: int) -> int:
    return pad_rows(rows) * (K // 16)


def tile_nvfp4_scales(s_code: np.ndarray) -> np.ndarray:
    rows, J = s_code.shape
    K = J * 16
    out = np.zeros(nvfp4_scales_bytes(rows, K), dtype=np.uint8)
    m, j = np.meshgrid(np.arange(rows), np.arange(J), indexing="ij")
    out[nvfp4_scale_offset(m, j, K)] = s_code
    return out


def untile_nvfp4_scales(tiled: np.ndarray, rows: int, K: int) -> np.ndarray:
    m, j = np.meshgrid(np.arange(rows), np.arange(K // 16), indexing="ij")
    return np.asarray(tiled, dtype=np.uint8)[nvfp4_scale_offset(m, j, K)]


# --------------------------------------------------------------- INT4 scales
def int4_scales_elems(rows: int, K: int) -> int:
    return (K // 64) * pad_rows(rows)


def tile_int4_scales(scales: np.ndarray) -> np.ndarray:
    """[rows, K/64] FP16 values -> [K/64, rows_pad] FP16 bits (uint16)."""
    rows, G = scales.shape
    out = np.zeros((G, pad_rows(rows)), dtype=np.float16)
    out[:, :rows] = np.asarray(scales, dtype=np.float64).T.astype(np.float16)
    return out.view(np.uint16).reshape(-1)


def untile_int4_scales(tiled: np.ndarray, rows: int, K: int) -> np.ndarray:
    t = np.asarray(tiled, dtype=np.uint16).reshape(K // 64, pad_rows(rows))
    return t[:, :rows].view(np.float16).astype(np.float64).T.copy()


# --------------------------------------------------------------- INT4 codes
def tile_int4_codes(q: np.ndarray) -> np.ndarray:
    """q [rows, K] integers in -7..7 -> tiled bytes [rows, K/2] (two's complement nibbles)."""
    q = np.asarray(q).astype(np.int16)
    if np.any(np.abs(q) > 7):
        raise ValueError("INT4 codes must lie in -7..7")
    nib = (q & 0xF).astype(np.uint8)  # v & 15
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def untile_int4_codes(tiled: np.ndarray) -> np.ndarray:
    """Tiled bytes [rows, K/2] -> q [rows, K] int16."""
    t = np.asarray(tiled, dtype=np.uint8)
    nib = np.empty(t.shape[:-1] + (t.shape[-1] * 2,), dtype=np.int16)
    nib[..., 0::2] = t & 0xF
    nib[..., 1::2] = t >> 4
    return np.where(nib >= 8, nib - 16, nib).astype(np.int16)


# --------------------------------------------------------------- AWQ qweight
_AWQ_SLOT_ROW = np.array([0, 8, 0, 8, 0, 8, 0, 8])
_AWQ_SLOT_COL = np.array([0, 0, 8, 8, 1, 1, 9, 9])


def awq_qweight_bytes(N: int, K: int) -> int:
    return pad_rows(N, 16) * K // 2


def tile_awq_qweight(q: np.ndarray) -> np.ndarray:
    """q [N, K] uint8 in 0..15 -> fragment-ordered bytes."""
    N, K = q.shape
    Np = pad_rows(N, 16)
    qp = np.zeros((Np, K), dtype=np.uint32)
    qp[:N] = q
    G = K // 64
    words = np.zeros((Np // 16, G, 32, 4), dtype=np.uint32)
    t = np.arange(32)
    r0, c0 = t // 4, 2 * (t % 4)
    for b in range(Np // 16):
        for g in range(G):
            for j in range(4):
                w = np.zeros(32, dtype=np.uint32)
                for s in range(8):
                    rows = b * 16 + r0 + _AWQ_SLOT_ROW[s]
                    cols = g * 64 + 16 * j + c0 + _AWQ_SLOT_COL[s]
                    w |= qp[rows, cols] << np.uint32(4 * s)
                words[b, g, :, j] = w
    return words.reshape(-1).view(np.uint8).copy()


def untile_awq_qweight(tiled: np.ndarray, N: int, K: int) -> np.ndarray:
    Np = pad_rows(N, 16)
    G = K // 64
    words = np.asarray(tiled, dtype=np.uint8).view(np.uint32).reshape(Np // 16, G, 32, 4)
    q = np.zeros((Np, K), dtype=np.uint8)
    t = np.arange(32)
    r0, c0 = t // 4, 2 * (t % 4)
    for b in range(Np // 16):
        for g in range(G):
            for j in range(4):
                w = words[b, g, :, j]
                for s in range(8):
                    rows = b * 16 + r0 + _AWQ_SLOT_ROW[s]
                    cols = g * 64 + 16 * j + c0 + _AWQ_SLOT_COL[s]
                    q[rows, cols] = (w >> np.uint32(4 * s)) & 0xF
    return q[:N]


# ------------------------------------------------------ AWQ scales and zeros
def tile_awq_sz(s_bits: np.ndarray, z_bits: np.ndarray) -> np.ndarray:
    """s, z [N, K/64] bf16 bits -> [N/16][K/64][16][2] bf16 bits."""
    N, G = s_bits.shape
    Np = pad_rows(N, 16)
    out = np.zeros((Np // 16, G, 16, 2), dtype=np.uint16)
    sp = np.zeros((Np, G), dtype=np.uint16)
    zp = np.zeros((Np, G), dtype=np.uint16)
    sp[:N], zp[:N] = s_bits, z_bits
    out[..., 0] = sp.reshape(Np // 16, 16, G).transpose(0, 2, 1)
    out[..., 1] = zp.reshape(Np // 16, 16, G).transpose(0, 2, 1)
    return out.reshape(-1)


def untile_awq_sz(tiled: np.ndarray, N: int, K: int):
    Np = pad_rows(N, 16)
    G = K // 64
    t = np.asarray(tiled, dtype=np.uint16).reshape(Np // 16, G, 16, 2)
    s = t[..., 0].transpose(0, 2, 1).reshape(Np, G)[:N]
    z = t[..., 1].transpose(0, 2, 1).reshape(Np, G)[:N]
    return s.copy(), z.copy()


# ------------------------------------------------------ down-projection operand
def lowrank_operand(L1: np.ndarray, smooth_inv: np.ndarray | None) -> np.ndarray:
    """L1 [K, r] (bf16 values), smooth_inv [K] (float32 values) -> [2, r, K] bf16 values."""
    from .formats import bf16_round, rn32
    v = np.asarray(L1, np.float64).T.copy()
    if smooth_inv is not None:
        v = rn32(v * np.asarray(smooth_inv, np.float64)[None, :])
    hi = bf16_round(v)
    lo = bf16_round(rn32(v - hi))
    return np.stack([hi, lo])
