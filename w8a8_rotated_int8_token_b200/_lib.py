"""ctypes view of libconvrot.so: one Python callable per C entry point, same names.

Loading fails loudly if the library has not been built; there is no other
implementation of these operations in this package.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libconvrot.so")

_c_void_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_size = ctypes.c_size_t

# name -> (restype, argtypes), mirroring include/convrot.h
SIGNATURES = {
    "convrot_abi_version": (_int, []),
    "convrot_status_string": (ctypes.c_char_p, [_int]),
    "convrot_prepare_weight_workspace_bytes": (_size, []),
    "convrot_prepare_weight": (_int, [_c_void_p, _i64, _i64, _int, _c_void_p, _c_void_p, _c_void_p, _size,
                                      _c_void_p]),
    "convrot_quant_act": (_int, [_c_void_p, _i64, _i64, _int, _c_void_p, _c_void_p, _c_void_p]),
    "convrot_linear_workspace_bytes": (_size, [_i64, _i64, _i64, _int]),
    "convrot_linear": (_int, [_c_void_p, _i64, _i64, _int, _c_void_p, _c_void_p, _i64, _c_void_p, _c_void_p,
                              _c_void_p, _size, _c_void_p]),
    "convrot_linear_timed": (_int, [_c_void_p, _i64, _i64, _int, _c_void_p, _c_void_p, _i64, _c_void_p,
                                    _c_void_p, _c_void_p, _size, _c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "convrot_linear_launch_count": (_int, [_i64, _i64, _i64, _int]),
    "convrot_linear_one_launch": (_int, [_c_void_p, _i64, _i64, _int, _c_void_p, _c_void_p, _i64, _c_void_p,
                                         _c_void_p, _c_void_p, _size, _c_void_p]),
    "convrot_prepare_weight_ex": (_int, [_c_void_p, _int, _i64, _i64, _int, _int, _c_void_p, _c_void_p, _c_void_p,
                                         _size, _c_void_p]),
    "convrot_quant_act_ex": (_int, [_c_void_p, _int, _i64, _i64, _i64, _int, _c_void_p, _c_void_p, _c_void_p]),
    "convrot_linear_ex": (_int, [_c_void_p, _int, _i64, _i64, _i64, _int, _c_void_p, _c_void_p, _int, _i64,
                                 _c_void_p, _c_void_p, _int, _c_void_p, _i64, _c_void_p, _size, _c_void_p]),
    "convrot_gemm_workspace_bytes": (_size, []),
    "convrot_gemm_dequant": (_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, _c_void_p,
                                    _c_void_p, _c_void_p, _size, _c_void_p]),
    "convrot_gemm_s32": (_int, [_c_void_p, _c_void_p, _i64, _i64, _i64, _c_void_p, _c_void_p, _size,
                                _c_void_p]),
    "convrot_linear_noalloc": (_int, [_c_void_p, _i64, _i64, _int, _c_void_p, _c_void_p, _i64, _c_void_p,
                                      _c_void_p, _c_void_p, _c_void_p]),
    "convrot_read_device_status": (_int, [_c_void_p, _c_void_p]),
    "convrot_test_wait_timeout": (_int, [_c_void_p, _size, _i64, _c_void_p]),
    "convrot_probe_i8_peak": (_int, [_i64, _c_void_p, _size, _c_void_p, _size, _c_void_p]),
    "convrot_attention_workspace_bytes": (_size, [_i64, _i64, _i64, _i64]),
    "convrot_attention_int8": (_int, [_c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, _i64, ctypes.c_float,
                                      _c_void_p, _c_void_p, _size, _c_void_p]),
    "convrot_probe_i8_peak_ctas": (_int, []),
    "convrot_probe_ex2_peak": (_int, [_i64, _c_void_p, _size, _c_void_p]),
    "convrot_probe_ex2_per_iter": (_i64, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libconvrot.so (once) and declare every entry point's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m w8a8_rotated_int8_token_b200.build` "
            "(the ConvRot operations exist only as CUDA kernels)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
