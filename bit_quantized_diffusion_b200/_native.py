"""ctypes declarations of the C ABI in include/svdq.h (libsvdq.so, built in-tree).

Loading fails loudly when the library is missing: there is no other
implementation of these calls in this package.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsvdq.so")

# status codes
OK, ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = range(6)
# formats / outputs / pack kinds
NVFP4_G16, INT4_G64 = 0, 1
OUT_BF16, OUT_F32 = 0, 1
PACK_ACT, PACK_WEIGHT, PACK_AWQ = 0, 1, 2

EXPORTS = (
    "svdq_status_str", "svdq_version", "svdq_codes_bytes", "svdq_scales_bytes",
    "awq_qweight_bytes", "awq_sz_bytes", "svdq_quantize_act", "svdq_w4a4_linear",
    "awq_w4a16_linear", "svdq_pack", "svdq_unpack", "svdq_check_device_status",
    "svdq_debug_wait_timeout", "svdq_pack_lowrank", "svdq_xl1_splits",
    "svdq_quantize_act_noalloc", "svdq_tensor_scale", "svdq_quantize_act_two_level",
    "svdq_w4a4_linear_two_level", "svdq_w4a4_linear_qkv_norm_rope",
    "svdq_column_absmax", "svdq_smoothing", "svdq_lowrank_factors", "svdq_residual",
    "awq_quantize_weight", "svdq_mlp_splits", "svdq_mlp_fc1",
)

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_S = ctypes.c_size_t


def load() -> ctypes.CDLL:
    """Load libsvdq.so and declare every exported signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m bit_quantized_diffusion_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "svdq_status_str": (ctypes.c_char_p, [_I]),
        "svdq_version": (_I, []),
        "svdq_codes_bytes": (_S, [_I, _I, _I]),
        "svdq_scales_bytes": (_S, [_I, _I, _I]),
        "awq_qweight_bytes": (_S, [_I, _I]),
        "awq_sz_bytes": (_S, [_I, _I]),
        "svdq_quantize_act": (_I, [_I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P]),
        "svdq_w4a4_linear": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P]),
        "awq_w4a16_linear": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
        "svdq_pack": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
        "svdq_unpack": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
        "svdq_check_device_status": (_I, [_P]),
        "svdq_debug_wait_timeout": (_I, [_I, _P]),
        "svdq_pack_lowrank": (_I, [_I, _I, _P, _P, _P, _P]),
        "svdq_xl1_splits": (_I, [_I, _I, _I]),
        "svdq_quantize_act_noalloc": (_I, [_I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P]),
        "svdq_tensor_scale": (_I, [_I, _I, _P, _I, _P, _P, _P]),
        "svdq_quantize_act_two_level": (_I, [_I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P]),
        "svdq_w4a4_linear_two_level": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                            _P, _I, _I, _P]),
        "svdq_w4a4_linear_qkv_norm_rope": (_I, [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                ctypes.c_float, _P, _P, _P, _I, _I, _P]),
        "svdq_column_absmax": (_I, [_I, _I, _P, _I, _P, _P]),
        "svdq_smoothing": (_I, [_I, _I, _P, _P, _P, _P]),
        "svdq_lowrank_factors": (_I, [_I, _I, _I, _P, _I, _P, _P, _I, _P, _P, _P]),
        "svdq_residual": (_I, [_I, _I, _I, _P, _P, _P, _P, _P, _P]),
        "awq_quantize_weight": (_I, [_I, _I, _P, _P, _P, _P]),
        "svdq_mlp_splits": (_I, [_I, _I]),
        "svdq_mlp_fc1": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


class SvdqError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = load().svdq_status_str(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != OK:
        raise SvdqError(status, where)
