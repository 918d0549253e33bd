"""ctypes declarations of libgptq_b200.so (the C ABI in include/gptq.h).

Loading fails loudly: there is no fallback implementation of any entry point.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptq_b200.so")
# the same library built with device-side index checks (gptq_device_checks)
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptq_b200_debug.so")

GPTQ_OK = 0
GPTQ_ERR_INVALID_ARG = 1
GPTQ_ERR_UNSUPPORTED = 2
GPTQ_ERR_WORKSPACE = 3
GPTQ_ERR_CUDA = 4
GPTQ_ERR_TIMEOUT = 5

GPTQ_BF16 = 0
GPTQ_F32 = 1

GPTQ_OP_HESSIAN = 0
GPTQ_OP_CHOLESKY = 1
GPTQ_OP_QUANTIZE = 2
GPTQ_OP_DEQUANT_MATVEC = 3

EXPORTS = ("gptq_workspace_size", "gptq_hessian_accumulate", "gptq_cholesky_inverse",
           "gptq_quantize_layer", "gptq_pack_int4", "gptq_pack_int3", "gptq_dequant",
           "gptq_status_string", "gptq_launch_count", "gptq_cholesky_inverse_noalloc",
           "gptq_selftest_division", "gptq_dequant_matvec", "gptq_gather_columns_u8",
           "gptq_hadamard_rows", "gptq_hadamard_cols", "gptq_set_wait_gate",
           "gptq_device_checks")


class GptqConfig(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group_size", ctypes.c_int),
                ("percdamp", ctypes.c_float), ("block", ctypes.c_int),
                ("actorder", ctypes.c_int), ("sym", ctypes.c_int)]


_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_int = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t

_SIGNATURES = {
    "gptq_workspace_size": (_int, [_int, _i64, _i64, _i64, _int, ctypes.POINTER(GptqConfig),
                                   ctypes.POINTER(_sz)]),
    "gptq_hessian_accumulate": (_int, [_vp, _vp, _int, _i64, _i64, _i64, _int, _f, _vp, _sz,
                                       _vp, _vp]),
    "gptq_cholesky_inverse": (_int, [_vp, _i64, _f, _int, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                                     _vp]),
    "gptq_quantize_layer": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _vp,
                                   ctypes.POINTER(GptqConfig), _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _sz, _vp, _vp, _vp]),
    "gptq_pack_int4": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "gptq_pack_int3": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "gptq_dequant": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _int, _i64, _vp, _vp, _int, _vp]),
    "gptq_status_string": (ctypes.c_char_p, [_int]),
    "gptq_launch_count": (_i64, []),
    "gptq_cholesky_inverse_noalloc": (_int, [_vp, _i64, _f, _int, _vp, _vp, _vp, _vp, _vp]),
    "gptq_selftest_division": (_int, [_vp, _vp, _i64, _vp, _vp]),
    "gptq_dequant_matvec": (_int, [_vp, _int, _i64, _i64, _vp, _vp, _int, _i64, _vp, _vp, _vp,
                                   _int, _i64, _vp, _vp, _sz, _vp]),
    "gptq_gather_columns_u8": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "gptq_hadamard_rows": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _int, _vp, _int, _i64, _vp]),
    "gptq_hadamard_cols": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _int, _vp, _int, _i64, _vp]),
    "gptq_set_wait_gate": (_int, [_vp, _i64]),
    "gptq_device_checks": (_int, [ctypes.POINTER(ctypes.c_uint32)]),
}

_LIB = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (once) and declare the library; raises if it is not built."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"{p} is missing: build it with `python -m post_weight_quantization_25_b200.build`"
            " (there is no non-CUDA implementation)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _LIB = lib
    return lib
