"""ctypes loader for libobgemm.so (the C ABI declared in include/obgemm.h).

There is no fallback: if the library is missing or cannot be loaded, importing
the ops raises, naming the build command.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libobgemm.so")

OB_OK = 0
STATUS_NAMES = {
    0: "OB_OK", 1: "OB_ERR_NULL", 2: "OB_ERR_SHAPE", 3: "OB_ERR_ALIGN", 4: "OB_ERR_NAN",
    5: "OB_ERR_NOT_CONVERGED", 6: "OB_ERR_WORKSPACE", 7: "OB_ERR_CUDA", 8: "OB_ERR_DEVICE_TIMEOUT",
    9: "OB_ERR_UNSUPPORTED", 10: "OB_ERR_DEVICE_BOUNDS",
}
OB_OUT_BF16, OB_OUT_F32 = 0, 1
OB_PATH_AUTO, OB_PATH_SIMT, OB_PATH_TC, OB_PATH_MMA_DECODE, OB_PATH_I8 = 0, 1, 3, 4, 5
OB_PATH_TC1 = 7  # the one-CTA tcgen05 GEMM even where the CTA pair applies
OB_PATH_STACK = 6  # dbf_linear only: both products in one persistent launch (M <= 16)
OB_FLAG_STATIC_WEIGHTS = 0x100  # OR into path: W_packed, a, b not written by the previous kernel



class ObLayer(ctypes.Structure):
    """struct ob_layer (include/obgemm.h): one layer of ob_linear_stack."""
    _fields_ = [("X", ctypes.c_void_p), ("W_packed", ctypes.c_void_p), ("a", ctypes.c_void_p),
                ("b", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("K", ctypes.c_int64), ("N", ctypes.c_int64),
                ("y_dtype", ctypes.c_int32), ("after_previous", ctypes.c_int32)]


# Every function the header declares, with (restype, argtypes).
_P, _I64, _I, _F, _SZ, _U64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                ctypes.c_size_t, ctypes.c_uint64)
SIGNATURES = {
    "ob_status_string": (ctypes.c_char_p, [_I]),
    "ob_version": (_I, []),
    "ob_last_device_error": (_I, [_P]),
    "ob_pack_signs": (_I, [_P, _I64, _I64, _P, _P]),
    "ob_svid_workspace_size": (_SZ, [_I64, _I64]),
    "ob_svid_rank1": (_I, [_P, _I64, _I64, _P, _P, _P, _I, _F, ctypes.POINTER(ctypes.c_int), _P, _SZ, _P]),
    "ob_linear": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _P, _I, _P]),
    "ob_linear_ex": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _P, _I, _I, _P]),
    "ob_linear_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "ob_linear_ws": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _P, _I, _P, _SZ, _I, _P]),
    "ob_linear_ln": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _P, _I, _F, _I, _P]),
    "ob_stack_workspace_size": (_SZ, []),
    "ob_linear_stack_workspace_size": (_SZ, [ctypes.POINTER(ObLayer), _I, _I64]),
    "ob_linear_stack": (_I, [ctypes.POINTER(ObLayer), _I, _I64, _P, _SZ, _P]),
    "ob_linear_stack_ex": (_I, [ctypes.POINTER(ObLayer), _I, _I64, _P, _SZ, _I, _P]),
    "dbf_workspace_size": (_SZ, [_I64, _I64]),
    "dbf_linear": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _I64, _P, _P, _P, _I, _P, _SZ, _P]),
    "dbf_linear_ex": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _I64, _P, _P, _P, _I, _P, _SZ, _I, _P]),
    "ob_selftest_timeout": (_I, [_U64, _P]),
    "dbf_linear_noalloc": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _I64, _P, _P, _P, _I, _P]),
    "dbf_factorize_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "dbf_factorize": (_I, [_P, _I64, _I64, _I64, _P, _I, _I, _I, _F, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ,
                           _P]),
}
DBF_NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024


class ObError(RuntimeError):
    """A libobgemm call returned a status other than OB_OK."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)} "
                         f"({lib().ob_status_string(status).decode()})")


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once); raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m binary_weight_gemm_b200.build` (nvcc, sm_100a)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def check(fn: str, status: int) -> None:
    if status != OB_OK:
        raise ObError(fn, status)
