"""ctypes declarations of libqlora_nf4.so (mirrors include/qlora_nf4.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  Loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libqlora_nf4.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "qlora_nf4.h")

STATUS = {
    0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_MISALIGNED",
    3: "QLORA_ERR_UNSUPPORTED_SHAPE", 4: "QLORA_ERR_CUDA", 5: "QLORA_ERR_TIMEOUT",
    6: "QLORA_ERR_DEVICE_CHECK", 7: "QLORA_ERR_WORKSPACE", 8: "QLORA_ERR_NO_DEVICE",
}
QLORA_OK = 0
QLORA_ERR_WORKSPACE = 7
NOALLOC_SCRATCH_BYTES = 16 << 20
QLORA_ERR_TIMEOUT = 5
DEVSTAT_TIMEOUT = 1
DEVSTAT_NONFINITE = 2
DEVSTAT_LAYOUT = 4


class QloraError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


class NF4Struct(ctypes.Structure):
    _fields_ = [
        ("codes", ctypes.c_void_p),
        ("q8", ctypes.c_void_p),
        ("step", ctypes.c_void_p),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
    ]


_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_u32 = ctypes.c_uint32
_f32 = ctypes.c_float
_sz = ctypes.c_size_t
_szp = ctypes.POINTER(ctypes.c_size_t)
_nf4p = ctypes.POINTER(NF4Struct)

SIGNATURES = {
    "qlora_version": (_int, []),
    "qlora_status_string": (ctypes.c_char_p, [_int]),
    "qlora_nf4_levels": (None, [ctypes.POINTER(ctypes.c_float)]),
    "qlora_nf4_bytes": (_sz, [_i64, _i64, _szp, _szp, _szp]),
    "qlora_nf4_single_bytes": (_sz, [_i64, _i64, _szp, _szp]),
    "qlora_nf4_quantize": (_int, [_vp, _i64, _i64, _nf4p, _vp]),
    "qlora_nf4_dequant": (_int, [_nf4p, _vp, _vp]),
    "qlora_linear_workspace_bytes": (_sz, [_i64, _i64, _i64, _int]),
    "qlora_linear_fwd": (_int, [_vp, _i64, _nf4p, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_fwd_ex": (_int, [_vp, _i64, _nf4p, _vp, _vp, _int, _f32, _vp, _f32, _vp, _vp, _vp, _sz,
                                   _vp]),
    "qlora_linear_dropout_workspace_bytes": (_sz, [_i64, _i64, _i64, _int]),
    "qlora_linear_fwd_noalloc": (_int, [_vp, _i64, _nf4p, _vp, _vp, _int, _f32, _vp, _vp, _vp]),
    "qlora_linear_bwd": (_int, [_vp, _vp, _vp, _i64, _nf4p, _vp, _vp, _int, _f32, _vp, _vp, _vp,
                                _vp, _sz, _vp]),
    "qlora_linear_bwd_ex": (_int, [_vp, _vp, _vp, _i64, _nf4p, _vp, _vp, _int, _f32, _vp, _f32, _int, _vp,
                                   _vp, _vp, _vp, _sz, _vp]),
    "qlora_nf4_merge": (_int, [_nf4p, _vp, _i64, _i64, _vp, _vp, _int, _f32, _vp, _vp]),
    "qlora_get_device_status": (_int, [_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "qlora_selftest_wait_timeout": (_int, [_u32, _vp]),
    "qlora_set_wait_limit_us": (_u32, [_u32]),
    "qlora_set_gemm_pairing": (_int, [_int]),
    "qlora_gemm_units": (_int, [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "qlora_profile_enable": (_int, [_int]),
    "qlora_profile_read": (_int, [_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float)]),
}

KERNEL_KINDS = ["quantize", "dequant", "prep", "project", "gemm_fwd", "gemm_dx",
                "grad", "skinny", "merge"]
PROFILE_CAP = 4096

_LIB = None


def header_symbols() -> list:
    """Function names declared in include/qlora_nf4.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


def lib():
    """Load the library (once).  Raises if it is missing: there is no fallback."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is not built; run `python -m bit_nf4_quantized_19_b200.build` "
            "(or __graft_entry__.build()).  There is no CPU fallback.")
    L = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _LIB = L
    return L


def check(code: int, where: str) -> None:
    if code != QLORA_OK:
        raise QloraError(code, where)
