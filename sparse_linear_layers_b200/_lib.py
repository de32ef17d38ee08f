"""ctypes binding of libsbl.so (the C ABI declared in include/sbl.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  If the shared library is missing this module raises at import
time; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsbl.so")

SBL_OK = 0
SBL_ERR_INVALID_ARG = 1
SBL_ERR_UNSUPPORTED = 2
SBL_ERR_NONFINITE = 3
SBL_ERR_CUDA = 4
SBL_ERR_TIMEOUT = 5
SBL_ERR_WORKSPACE = 6

SBL_PREP_SCALE_BF16 = 1
SBL_PREP_SCALE_GLOBAL = 2

SBL_BWD_DW_TERNARY = 1

SBL_MAX_GROUP = 8

SBL_F32 = 0
SBL_BF16 = 1

SBL_PATH_AUTO = 0
SBL_PATH_DECODE = 1
SBL_PATH_PREFILL = 2
SBL_PATH_PREFILL_1CTA = 3
SBL_PATH_PREFILL_PAIR = 4
SBL_PATH_PREFILL_SPARSE = 5

# name -> (restype, argtypes); mirrors include/sbl.h
_vp, _i64, _int, _sz, _u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint32
_f32 = ctypes.c_float
SIGNATURES = {
    "sbl_prepare_weights": (_int, [_vp, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp]),
    "sbl_prepare_weights_ex": (_int, [_vp, _i64, _i64, _int, _int, _vp, _vp, _vp, _int, _vp]),
    "sbl_prepare_weights_grouped": (_int, [_int, _vp, _vp, _i64, _int, _int, _vp, _vp, _vp, _vp]),
    "sbl_quant_act": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "sbl_rmsnorm_quant_act": (_int, [_vp, _vp, _f32, _i64, _i64, _vp, _vp, _vp]),
    "sbl_linear_workspace_bytes": (_sz, [_i64, _i64, _i64, _int, _int]),
    "sbl_linear": (_int, [_vp, _i64, _i64, _vp, _vp, _i64, _int, _int, _vp, _int, _vp, _vp, _sz, _vp]),
    "sbl_linear_path": (_int, [_vp, _i64, _i64, _vp, _vp, _i64, _int, _int, _vp, _int, _vp, _vp, _sz, _int, _vp]),
    "sbl_linear_rmsnorm": (_int, [_vp, _vp, _f32, _i64, _i64, _vp, _vp, _i64, _int, _int, _vp, _int, _vp, _vp, _sz,
                                  _int, _vp]),
    "sbl_linear_q": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _i64, _int, _int, _vp, _int, _vp, _vp, _sz, _vp]),
    "sbl_linear_grouped_workspace_bytes": (_sz, [_i64, _i64]),
    "sbl_linear_grouped": (_int, [_vp, _i64, _i64, _int, _vp, _vp, _vp, _int, _int, _vp, _int, _vp, _vp, _sz, _vp]),
    "sbl_linear_noalloc": (_int, [_vp, _i64, _i64, _vp, _vp, _i64, _int, _int, _vp, _int, _vp, _vp]),
    "sbl_copy_to_device": (_int, [_vp, _vp, _sz, _vp]),
    "sbl_copy_to_host": (_int, [_vp, _vp, _sz, _vp]),
    "sbl_linear_hostio": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _int, _int, _vp, _vp, _int, _vp, _sz, _vp]),
    "sbl_linear_plan": (_int, [_i64, _i64, _i64, _int, _int, _sz]),
    "sbl_mask_monitor": (_int, [_vp, _vp, _i64, _i64, _int, _int, _vp, _vp, _vp]),
    "sbl_linear_backward": (_int, [_vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _int, _vp]),
    "sbl_linear_backward_workspace_bytes": (_sz, [_i64, _i64, _i64, _int, _int]),
    "sbl_linear_backward_ws": (_int, [_vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _int, _vp, _sz, _vp]),
    "sbl_decode_max_tokens": (_i64, []),
    "sbl_device_status": (_int, [_vp]),
    "sbl_selftest_bounded_wait": (_int, [_u32, _vp]),
    "sbl_status_string": (ctypes.c_char_p, [_int]),
    "sbl_version": (ctypes.c_char_p, []),
}


class SblError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libsbl.so not found at {LIB_PATH}; build it with `python -m sparse_linear_layers_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def status_string(code: int) -> str:
    return lib.sbl_status_string(code).decode()


def check(code: int, where: str) -> None:
    if code != SBL_OK:
        raise SblError(code, where)
