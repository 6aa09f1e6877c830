"""The fused QKV projection's epilogue, written plainly in float64.

ORACLE -- test infrastructure only. Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the product package
never does.

What it computes (Diffusers blog, the section on fused QKV: the three attention
projections joined into one ``to_qkv`` linear whose output dimension is Q, then
K, then V; the attention code splits each of Q and K into heads, applies
``norm_q`` / ``norm_k`` to every head and then the rotary embedding; Nunchaku
does all of this in one fused call on the projection's output):

    y        = the SVDQ layer's output [M, 3 H D]   (columns Q | K | V, D = 128)
    Q, K     : for each row m and head h, with v = y[m, head columns]
                 z = v / sqrt(mean(v^2) + eps) * gamma        (RMS norm of the head)
                 out[2i]   = z[2i] cos(theta[m, i]) - z[2i+1] sin(theta[m, i])
                 out[2i+1] = z[2i+1] cos(theta[m, i]) + z[2i] sin(theta[m, i])
    V        : unchanged

The pages show the calls, not their arithmetic; the readings this follows:
the norm is an RMS norm over each head's D = 128 values (FLUX's 3072 = 24 x
128), with a weight gamma [D] per projection (Q's and K's) and eps added to
the mean square; the rotation acts on adjacent pairs (2i, 2i+1) with one angle
per row and pair, given as tables cos, sin [M, D/2]; the norm comes before the
rotation, as in the attention code; and the whole epilogue is exact here (the
kernel computes it in float32 from its accumulator and rounds once, at the
output).
"""

from __future__ import annotations

import numpy as np

HEAD_DIM = 128


def rms_norm_heads(v: np.ndarray, gamma: np.ndarray | None, eps: float) -> np.ndarray:
    """v [M, heads, D] -> v / sqrt(mean over D of v^2 + eps) * gamma."""
    v = np.asarray(v, np.float64)
    ms = np.mean(v * v, axis=-1, keepdims=True)
    z = v / np.sqrt(ms + float(eps))
    if gamma is not None:
        z = z * np.asarray(gamma, np.float64)[None, None, :]
    return z


def rotate_pairs(z: np.ndarray, cos: np.ndarray | None, sin: np.ndarray | None) -> np.ndarray:
    """z [M, heads, D]; cos, sin [M, D/2]: pair (2i, 2i+1) of row m turned by angle i of row m."""
    z = np.asarray(z, np.float64)
    if cos is None:
        return z.copy()
    c = np.asarray(cos, np.float64)[:, None, :]
    s = np.asarray(sin, np.float64)[:, None, :]
    even, odd = z[..., 0::2], z[..., 1::2]
    out = np.empty_like(z)
    out[..., 0::2] = even * c - odd * s
    out[..., 1::2] = odd * c + even * s
    return out


def qkv_norm_rope(y: np.ndarray, heads: int, norm_q: np.ndarray | None, norm_k: np.ndarray | None,
                  eps: float, cos: np.ndarray | None, sin: np.ndarray | None) -> np.ndarray:
    """y [M, 3 heads D] (the projection's float64 output) -> the epilogue's output, float64."""
    y = np.asarray(y, np.float64)
    M, N = y.shape
    D = HEAD_DIM
    if N != 3 * heads * D:
        raise ValueError(f"{N} columns are not Q, K, V of {heads} heads of {D}")
    out = y.copy()
    for part, gamma in ((0, norm_q), (1, norm_k)):
        cols = slice(part * heads * D, (part + 1) * heads * D)
        v = y[:, cols].reshape(M, heads, D)
        out[:, cols] = rotate_pairs(rms_norm_heads(v, gamma, eps), cos, sin).reshape(M, heads * D)
    return out
