"""ctypes declarations of libqlora's C ABI (include/qlora.h).

Loading fails loudly: if the shared library is missing there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlora.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_SHAPE = 2
ERR_ALIGNMENT = 3
ERR_NONFINITE = 4
ERR_UNSUPPORTED = 5
ERR_CUDA = 6
ERR_TIMEOUT = 7
ERR_WORKSPACE = 8

FMT_NF4_DQ = 0
FMT_NF4_FP32SCALE = 1
FMT_AFFINE = 2
COMPUTE_FP32 = 0
COMPUTE_BF16 = 1
OP_FWD = 0
OP_BWD = 1


class qlora_weight(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("O", ctypes.c_int64),
        ("I", ctypes.c_int64),
        ("block", ctypes.c_int32),
        ("group", ctypes.c_int32),
        ("bits", ctypes.c_int32),
        ("codes", ctypes.c_void_p),
        ("scale_codes", ctypes.c_void_p),
        ("group_absmax", ctypes.c_void_p),
        ("mean", ctypes.c_void_p),
        ("scale", ctypes.c_void_p),
        ("bias", ctypes.c_void_p),
    ]


# name -> (restype, argtypes)
_P = ctypes.c_void_p
_W = ctypes.POINTER(qlora_weight)
_i64, _i32, _u32, _f32, _sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_nf4_codebook": (ctypes.c_int, [_P]),
    "qlora_nf4_payload_bytes": (_sz, [_i64, _i32, _i32]),
    "qlora_quantize_nf4_workspace_bytes": (_sz, [_i64, _i32, _i32]),
    "qlora_quantize_nf4": (ctypes.c_int, [_P, _i64, _i64, _i32, _i32, _P, _P, _P, _P, _P, _sz, _P]),
    "qlora_quantize_nf4_noalloc": (ctypes.c_int, [_P, _i64, _i64, _i32, _i32, _P, _P, _P, _P, _P]),
    "qlora_nf4_fp32scale_payload_bytes": (_sz, [_i64, _i32]),
    "qlora_quantize_nf4_fp32scale_workspace_bytes": (_sz, [_i64, _i32]),
    "qlora_quantize_nf4_fp32scale": (ctypes.c_int, [_P, _i64, _i64, _i32, _P, _P, _P, _sz, _P]),
    "qlora_quantize_affine_workspace_bytes": (_sz, [_i64, _i32, _i32]),
    "qlora_quantize_affine": (ctypes.c_int, [_P, _i64, _i64, _i32, _i32, _P, _P, _P, _P, _sz, _P]),
    "qlora_dequantize": (ctypes.c_int, [_W, _P, _P]),
    "qlora_merge": (ctypes.c_int, [_W, _P, _P, _i32, _f32, _P, _P]),
    "qlora_adam_step": (ctypes.c_int, [_P, _P, _P, _P, _i64, _i64, _f32, _f32, _f32, _f32, _i64, _P]),
    "qlora_linear_workspace_bytes": (_sz, [_W, _i64, _i32, _i32, _i32]),
    "qlora_linear_fwd": (ctypes.c_int, [_W, _P, _i64, _P, _P, _i32, _f32, _i32, _P, _P, _P, _sz, _P]),
    "qlora_linear_bwd": (ctypes.c_int, [_W, _P, _P, _i64, _P, _P, _i32, _f32, _P, _i32, _P, _P, _P, _P,
                                        _sz, _P]),
    "qlora_workspace_status": (ctypes.c_int, [_P, _P]),
    "qlora_selftest_wait_timeout": (ctypes.c_int, [_P, _sz, _u32, _P]),
    "qlora_kernel_launch_count": (ctypes.c_uint64, []),
    "qlora_kernel_timing_enable": (ctypes.c_int, [_i32]),
    "qlora_kernel_timing_collect": (ctypes.c_int32, [_P, _P, _P, _i32]),
}

_lib = None


def load() -> ctypes.CDLL:
    """The loaded library; raises if libqlora.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libqlora.so not built at {LIB_PATH}; run qlora_bit_frozen_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
